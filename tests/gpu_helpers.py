"""Helpers for the GPU parity tests: move a workload to the device, run one
engine step through the C-ABI binding, and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# spec tolerances for attention outputs (bf16 in, fp32 accumulation, bf16 out)
MAX_ABS = 1e-2
REL_L2 = 5e-3


def load_library() -> str:
    """Compile the in-tree libpa.so if it is missing or older than its sources
    (nvcc, about 30 s), then load it; raises if it cannot be built."""
    from paged_kv_cache_445_b200.csrc import build as pabuild
    pabuild.build()
    import paged_kv_cache_445_b200 as pa
    return pa.library_path  # touching a binding name loads the library


def bf16_to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def dev_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def i32(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


class DeviceStep:
    """A workload resident on the GPU, plus its workspace and status word."""

    def __init__(self, w, device="cuda"):
        import paged_kv_cache_445_b200 as pa
        self.w = w
        self.k_cache = bf16_to_dev(w.k_cache, device)
        self.v_cache = bf16_to_dev(w.v_cache, device)
        self.k_new = bf16_to_dev(w.k_new, device)
        self.v_new = bf16_to_dev(w.v_new, device)
        self.q = bf16_to_dev(w.q, device)
        self.block_tables = i32(w.block_tables, device)
        self.context_lens = i32(w.context_lens, device)
        self.query_start = i32(w.query_start, device)
        self.slot_mapping = i32(w.slot_mapping, device)
        self.out = torch.empty_like(self.q)
        self.workspace = pa.make_workspace(w.num_query_tokens, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                           w.block_tables.shape[1], w.block_size, device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def append(self):
        import paged_kv_cache_445_b200 as pa
        pa.pa_cache_append(self.k_new, self.v_new, self.k_cache, self.v_cache, self.slot_mapping, self.status)

    def attend(self, force_varlen=False):
        import paged_kv_cache_445_b200 as pa
        if self.w.is_decode and not force_varlen:
            pa.pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.block_tables, self.context_lens,
                         self.w.scale, self.workspace, self.status)
        else:
            pa.pa_prefill_chunk(self.out, self.q, self.query_start, self.k_cache, self.v_cache, self.block_tables,
                                self.context_lens, self.w.scale, self.workspace, self.status)

    def step(self, force_varlen=False):
        self.append()
        self.attend(force_varlen)
        torch.cuda.synchronize()
        return self.out.float().cpu().numpy()


def oracle_after_append(w):
    """Host copies of the caches after the oracle's own append."""
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    slots = oracle.slot_mapping(w.block_tables, w.context_lens, w.query_start, w.block_size, w.num_blocks)
    oracle.cache_append(w.k_new, w.v_new, kc, vc, slots)
    return kc, vc


def compare(got: np.ndarray, want: np.ndarray, what: str = ""):
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got.astype(np.float64) - want)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(err)) / denom if denom > 0 else float(np.linalg.norm(err))
    assert max_abs <= MAX_ABS, f"{what}: max abs error {max_abs:.3e} > {MAX_ABS}"
    assert rel <= REL_L2, f"{what}: relative L2 error {rel:.3e} > {REL_L2}"
    return max_abs, rel
