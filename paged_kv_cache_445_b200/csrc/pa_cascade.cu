// pa_cascade.cu -- the shared-prefix pass of decode attention: the query rows
// of every sequence in a group that shares a prefix of the KV cache attend to
// that prefix together, reading each of its K/V tiles once.
//
// What it computes: copy-on-write sharing stores a prompt's prefix once and
// lets all rollouts (or requests) of the prompt reference the same physical
// blocks ("vLLM serving internals", AI Engineering from Scratch, Phase 17 /
// 04, "PagedAttention as a virtual memory system"; "How vLLM gets real
// throughput on H100s", "PagedAttention borrows from operating systems": GRPO
// rollouts share the prompt's pages).  Softmax attention over keys 0..p splits
// exactly into the prefix keys and the rest: with m = max over all scores,
//   out = (sum_prefix e^(s - m) V + sum_rest e^(s - m) V) / (sum_prefix e^(s - m) + sum_rest e^(s - m)).
// This kernel produces, for every (sequence, query head) of a group and every
// slice of the prefix, the unnormalised partial (O = sum e^(s - m_k) V,
// m_k, l = sum e^(s - m_k)), m_k in log2 units; the decode kernel adds the private
// keys and folds these partials in before it normalises.
//
// How (B200): one M-tile = up to 128 rows = t sequences of a group x the G
// query heads of one KV head (t G a multiple of 8) (q rows of consecutive sequences are
// consecutive, so one 3-D TMA box per 64 head-dim columns brings them), N-tile
// = 64 prefix keys; S = Q K^T and O += P V on tcgen05 with S (double-buffered)
// and O in tensor memory, P written over S as the A operand of P V; a TMA
// warp, an MMA warp and a 128-thread softmax warpgroup (thread = row).  The
// prefix of each group is cut into up to CASCADE_SPLITS slices so that groups
// x KV heads x slices fill the GPU.  Every wait is bounded.
#include <cuda.h>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_umma.cuh"

namespace pa {

namespace {

constexpr int CS_THREADS = 192;
constexpr int CS_M = 128;  // rows per M-tile
constexpr int CS_N = 64;   // keys per tile
constexpr int CS_KST = 3;  // K stages
constexpr int CS_VST = 2;  // V stages
constexpr float CS_RESCALE_LOG2 = 8.f;

template <int D>
struct CascadeShape {
  static constexpr int PANELS = D / 64;                // 64-column (128-byte) panels of the head dim
  static constexpr int Q_PANEL = CS_M * 128;           // 16 KB
  static constexpr int KV_PANEL = CS_N * 128;          // 8 KB
  static constexpr int Q_BYTES = PANELS * Q_PANEL;
  static constexpr int KV_BYTES = PANELS * KV_PANEL;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = Q_BYTES;
  static constexpr int SMEM_V = SMEM_K + CS_KST * KV_BYTES;
  static constexpr int SMEM_TOTAL = SMEM_V + CS_VST * KV_BYTES;  // 224 KB at D = 256
  // S0 [0, 64), S1 [64, 128), P0 [128, 160), P1 [160, 192), O [256, 256 + D) (D = 64: [192, 256)).
  // P has buffers of its own: an MMA that writes S must never overwrite columns an earlier P V may
  // still be reading.  O starts on a multiple of its own width (up to 256 columns).
  static constexpr uint32_t TMEM_P = 2 * CS_N;
  static constexpr uint32_t TMEM_O = D <= 64 ? 192 : 256;
  static constexpr uint32_t TMEM_COLS = TMEM_O + D <= 256 ? 256 : 512;
};

struct CItem {
  int s0, ge;          // first sequence of the M-tile, end of the group
  int kvh, split;
  int t0, nt;          // prefix tiles [t0, t0 + nt) of 64 keys
  int table_seq;       // the group's first sequence: its table holds the shared blocks
};

struct CShared {
  uint64_t q_full, q_empty, o_empty, pv_done, p_full, drain;
  uint64_t s_full[2];
  uint64_t k_full[CS_KST], k_empty[CS_KST], v_full[CS_VST], v_empty[CS_VST];
  uint32_t tmem_base;
  int abort;
  long long total;
};

}  // namespace

// Items = (group, M-tile, KV head, prefix slice), group by group.
__device__ __forceinline__ bool cascade_item(const CascadeParams& p, int tokm, long long idx, CItem& it,
                                             long long* total_out) {
  long long base = 0;
  for (int g = 0; g < p.num_groups; ++g) {
    const int gs = __ldg(p.group_start + g), ge = __ldg(p.group_start + g + 1);
    const int span = cascade_span(__ldg(p.group_prefix + g));
    if (ge <= gs || span == 0) continue;
    const int ptiles = span / CS_N, nsplit = cascade_splits(span);
    const int tps = (ptiles + nsplit - 1) / nsplit;
    const int mtiles = (ge - gs + tokm - 1) / tokm;
    const long long n = static_cast<long long>(mtiles) * p.num_kv_heads * nsplit;
    if (!total_out && idx < base + n) {
      long long r = idx - base;
      it.split = static_cast<int>(r % nsplit);
      r /= nsplit;
      it.kvh = static_cast<int>(r % p.num_kv_heads);
      const int mt = static_cast<int>(r / p.num_kv_heads);
      it.s0 = gs + mt * tokm;
      it.ge = ge;
      it.table_seq = gs;
      it.t0 = it.split * tps;
      it.nt = min(tps, ptiles - it.t0);
      return true;
    }
    base += n;
  }
  if (total_out) *total_out = base;
  return false;
}

__device__ __forceinline__ bool cs_wait(CShared& sh, uint64_t* bar, uint32_t phase, int* status) {
  if (mbar_try_wait(bar, phase)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t polls = 0;; ++polls) {
    if (mbar_try_wait(bar, phase)) return true;
    if ((polls & 63) == 0) {
      if (*reinterpret_cast<volatile int*>(&sh.abort)) return false;
      if (globaltimer_ns() - t0 > WAIT_NS) {
        sh.abort = 1;
        set_status(status, PA_STATUS_BIT(PA_ERR_TIMEOUT));
        return false;
      }
    }
  }
}

// A wait taken by a whole warp: one answer for all its lanes, so the warp
// stays converged for the predicated MMA issue or the warp-collective
// tensor-memory loads and stores that follow.
__device__ __forceinline__ bool cs_wait_warp(CShared& sh, uint64_t* bar, uint32_t phase, int* status) {
  return __all_sync(FULL_MASK, cs_wait(sh, bar, phase, status));
}

template <int D>
__global__ void __launch_bounds__(CS_THREADS, 1)
    cascade_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv, const CascadeParams p) {
  using S = CascadeShape<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ CShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;
  const int tokm = cascade_tokm(G);  // sequences per M-tile

  if (threadIdx.x == 0) {
    mbar_init(&sh.q_full, 1);
    mbar_init(&sh.q_empty, 1);
    mbar_init(&sh.o_empty, 128);
    mbar_init(&sh.pv_done, 1);
    mbar_init(&sh.p_full, 128);
    mbar_init(&sh.drain, 1);
    for (int b = 0; b < 2; ++b) mbar_init(&sh.s_full[b], 1);
    for (int b = 0; b < CS_KST; ++b) {
      mbar_init(&sh.k_full[b], 1);
      mbar_init(&sh.k_empty[b], 1);
    }
    for (int b = 0; b < CS_VST; ++b) {
      mbar_init(&sh.v_full[b], 1);
      mbar_init(&sh.v_empty[b], 1);
    }
    sh.abort = 0;
    CItem unused;
    cascade_item(p, tokm, 0, unused, &sh.total);
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh.tmem_base)),
                 "r"(S::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  grid_dependency_wait();  // the cache may still be being written by the kernel before this one
  const long long total = sh.total;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmq);
      prefetch_tmap(&tmk);
      prefetch_tmap(&tmv);
    }
    const uint64_t pol = policy_evict_last();  // every M-tile and KV head of a group re-reads the prefix
    const uint32_t q_bytes = static_cast<uint32_t>(S::PANELS) * 128u * static_cast<uint32_t>(G * tokm);
    uint32_t items = 0, tcount = 0;
    for (long long idx = blockIdx.x; idx < total && !sh.abort; idx += gridDim.x, ++items) {
      CItem it;
      if (!cascade_item(p, tokm, idx, it, nullptr)) break;
      const int32_t* table = p.block_tables + static_cast<long long>(it.table_seq) * p.max_blocks;
      if (items > 0 && !cs_wait(sh, &sh.q_empty, (items - 1) & 1, p.status)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&sh.q_full, q_bytes);
#pragma unroll
        for (int pc = 0; pc < S::PANELS; ++pc)
          tma_load_3d(smem + S::SMEM_Q + pc * S::Q_PANEL, &tmq, &sh.q_full, pc * 64, it.kvh * G, it.s0);
      }
      auto load_tile = [&](const CUtensorMap* tm, uint64_t* full, uint64_t* empty, int nst, int base_off,
                           uint32_t t, int j) -> bool {
        const int st = t % nst;
        const uint32_t use = t / nst;
        if (use > 0 && !cs_wait(sh, &empty[st], (use - 1) & 1, p.status)) return false;
        if (lane == 0) mbar_arrive_expect_tx(&full[st], S::KV_BYTES);
        __syncwarp();
        if (lane < CS_N / 16) {  // lane b: keys 16b.. of the tile, every head-dim panel
          const int key0 = (it.t0 + j) * CS_N + lane * 16;
          const int lb = key0 / p.block_size, y = key0 - lb * p.block_size;
          const int blk = lb < p.max_blocks ? __ldg(table + lb) : -1;
          if (blk < 0 || blk >= p.num_blocks) set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
          uint8_t* dst = smem + base_off + st * S::KV_BYTES + lane * 2048;
#pragma unroll
          for (int pc = 0; pc < S::PANELS; ++pc)
            tma_load_4d(dst + pc * S::KV_PANEL, tm, &full[st], pc * 64, y, it.kvh, blk, pol);
        }
        return true;
      };
      bool ok = true;
      for (int j = 0; ok && j < it.nt; ++j) {
        ok = load_tile(&tmk, sh.k_full, sh.k_empty, CS_KST, S::SMEM_K, tcount + j, j);
        if (ok && j > 0) ok = load_tile(&tmv, sh.v_full, sh.v_empty, CS_VST, S::SMEM_V, tcount + j - 1, j - 1);
      }
      if (ok) ok = load_tile(&tmv, sh.v_full, sh.v_empty, CS_VST, S::SMEM_V, tcount + it.nt - 1, it.nt - 1);
      tcount += it.nt;
      if (!ok) break;
    }
    if (sh.abort) {  // let copies in flight land before shared memory goes away
      for (int st = 0; st < CS_KST; ++st) {
        const uint32_t uses = tcount / CS_KST + (static_cast<uint32_t>(st) < tcount % CS_KST ? 1u : 0u);
        if (uses > 0) mbar_wait(&sh.k_full[st], (uses - 1) & 1);
      }
      for (int st = 0; st < CS_VST; ++st) {
        const uint32_t uses = tcount / CS_VST + (static_cast<uint32_t>(st) < tcount % CS_VST ? 1u : 0u);
        if (uses > 0) mbar_wait(&sh.v_full[st], (uses - 1) & 1);
      }
      if (items > 0) mbar_wait(&sh.q_full, (items - 1) & 1);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    const uint32_t idesc_qk = umma_idesc(CS_M, CS_N, 0, 0);
    constexpr int PV_N = D < 128 ? D : 128;  // P V in column blocks of at most 128 (two MMAs at head_dim 256)
    const uint32_t idesc_pv = umma_idesc(CS_M, PV_N, 0, 1);
    const uint32_t sq = smem_u32(smem + S::SMEM_Q);
    uint32_t q_phase = 0, p_phase = 0, o_phase = 0, kv_count = 0;
    bool first_item = true;
    for (long long idx = blockIdx.x; idx < total && !sh.abort; idx += gridDim.x) {
      CItem it;
      if (!cascade_item(p, tokm, idx, it, nullptr)) break;
      const int nt = it.nt;
      if (!cs_wait_warp(sh, &sh.q_full, q_phase, p.status)) break;
      q_phase ^= 1;
      if (!first_item) {  // the epilogue of the previous item has read O
        if (!cs_wait_warp(sh, &sh.o_empty, o_phase, p.status)) break;
        o_phase ^= 1;
      }
      first_item = false;
      // S(j) into buffer j & 1: its previous tile was read by the softmax before
      // it handed over P(j - 2), and no MMA reads S
      auto qk = [&](int j) -> bool {
        const int stage = (kv_count + j) % CS_KST;
        if (!cs_wait_warp(sh, &sh.k_full[stage], ((kv_count + j) / CS_KST) & 1, p.status)) return false;
        tc_fence_after();
        const uint32_t sk = smem_u32(smem + S::SMEM_K + stage * S::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_f16(tmem + (j & 1) * CS_N, umma_desc(sq + (kk >> 2) * S::Q_PANEL + (kk & 3) * 32, 16, 1024),
                   umma_desc(sk + (kk >> 2) * S::KV_PANEL + (kk & 3) * 32, 16, 1024), idesc_qk, kk > 0);
        umma_commit(&sh.s_full[j & 1]);
        umma_commit(&sh.k_empty[stage]);
        if (j == nt - 1) umma_commit(&sh.q_empty);
        return true;
      };
      auto pv = [&](int j) -> bool {
        if (!cs_wait_warp(sh, &sh.p_full, p_phase, p.status)) return false;
        p_phase ^= 1;
        const int stage = (kv_count + j) % CS_VST;
        if (!cs_wait_warp(sh, &sh.v_full[stage], ((kv_count + j) / CS_VST) & 1, p.status)) return false;
        tc_fence_after();
        const uint32_t sv = smem_u32(smem + S::SMEM_V + stage * S::KV_BYTES);
#pragma unroll
        for (int nb = 0; nb < D / PV_N; ++nb)  // O columns [PV_N nb, PV_N (nb + 1)): V panels 2 nb, 2 nb + 1
#pragma unroll
          for (int kk = 0; kk < CS_N / 16; ++kk)  // keys 16kk..: P columns 8kk.., V rows 16kk..
            umma_f16_ts(tmem + S::TMEM_O + nb * PV_N, tmem + S::TMEM_P + (j & 1) * (CS_N / 2) + 8 * kk,
                        umma_desc(sv + nb * (PV_N / 64) * S::KV_PANEL + kk * 16 * 128, S::KV_PANEL, 1024), idesc_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&sh.pv_done);
        umma_commit(&sh.v_empty[stage]);
        return true;
      };
      bool ok = qk(0);
      for (int j = 1; ok && j < nt; ++j) ok = qk(j) && pv(j - 1);
      if (ok) ok = pv(nt - 1);
      kv_count += nt;
      if (!ok) break;
    }
  } else {
    // ================================================================ softmax warpgroup
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const int seq_off = row / G, head = row % G;
    const float cs = p.scale_log2;
    // pv_count: completions of pv_done before this item (one per P V).  The
    // softmax waits for every one of them, in order: a parity wait is exact
    // only when the previous phase is known to have completed.
    uint32_t s_phase[2] = {0, 0}, pv_count = 0;
    for (long long idx = blockIdx.x; idx < total && !sh.abort; idx += gridDim.x) {
      CItem it;
      if (!cascade_item(p, tokm, idx, it, nullptr)) break;
      const int nt = it.nt;
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nt && ok; ++j) {
        const int sb = j & 1;
        if (!(ok = cs_wait_warp(sh, &sh.s_full[sb], s_phase[sb], p.status))) break;
        s_phase[sb] ^= 1;
        tc_fence_after();
        float s[CS_N];
#pragma unroll
        for (int c = 0; c < CS_N / 32; ++c) {
          float v[32];
          tmem_ld32(tmem + lane_addr + sb * CS_N + c * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = v[i];
        }
        tmem_wait_ld();
        // every prefix key is visible to every row: the largest scaled score is
        // cs * (max raw score), or cs * (min raw score) for a negative scale
        float m8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = s[k];
        if (cs >= 0.f) {
#pragma unroll
          for (int i = 8; i < CS_N; i += 8)
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = fmaxf(m8[k], s[i + k]);
        } else {
#pragma unroll
          for (int i = 8; i < CS_N; i += 8)
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = fminf(m8[k], s[i + k]);
        }
        float mr = m8[0];
#pragma unroll
        for (int k = 1; k < 8; ++k) mr = cs >= 0.f ? fmaxf(mr, m8[k]) : fminf(mr, m8[k]);
        const float mxs = cs * mr;
        const bool rescale = mxs > m_ref + CS_RESCALE_LOG2 || m_ref == -INFINITY;
        const float m_new = rescale ? fmaxf(mxs, m_ref) : m_ref;
        const float neg_m = -m_new;
        uint32_t pk[32];
        float l8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float a = fast_exp2(fmaf(s[2 * i], cs, neg_m));
          const float b = fast_exp2(fmaf(s[2 * i + 1], cs, neg_m));
          l8[i & 7] += a + b;
          pk[i] = pack_bf16x2(a, b);
        }
        const bool resc = rescale && m_ref != -INFINITY;
        const float alpha = resc ? fast_exp2(m_ref - m_new) : 1.f;
        l = l * alpha + (((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7])));
        m_ref = m_new;
        if (j > 0) {
          // P V(j - 1) (phase pv_count + j - 1; P V(j - 2) was waited for at tile
          // j - 1, and P V(j) needs this tile's P) must be done before O is
          // rescaled and before P buffer j & 1, last read by P V(j - 2), is rewritten
          if (!(ok = cs_wait_warp(sh, &sh.pv_done, (pv_count + j - 1) & 1, p.status))) break;
          tc_fence_after();
          // scale O (warp-uniform: tcgen05.ld/st are warp-collective; rows that
          // keep their max scale by 1)
          if (__any_sync(FULL_MASK, resc)) {
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              float v[32];
              tmem_ld32(tmem + lane_addr + S::TMEM_O + c * 32, v);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= alpha;
              tmem_st32(tmem + lane_addr + S::TMEM_O + c * 32, v);
            }
          }
        }
        tmem_st32u(tmem + lane_addr + S::TMEM_P + sb * (CS_N / 2), pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sh.p_full);
      }
      pv_count += nt;
      if (!ok) break;
      // ---- epilogue: the unnormalised partial of this row and prefix slice
      if (!cs_wait_warp(sh, &sh.pv_done, (pv_count - 1) & 1, p.status)) break;
      tc_fence_after();
      const int seq = it.s0 + seq_off;
      const bool valid = seq_off < tokm && seq < it.ge;
      float* dst = p.partials + ((static_cast<long long>(valid ? seq : 0) * p.num_q_heads + it.kvh * G + head) *
                                     (CASCADE_SPLITS + 1) + it.split) * cascade_record_floats(D);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_addr + S::TMEM_O + c * 32, v);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + c * 32 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
      }
      if (valid) {
        dst[D] = m_ref;
        dst[D + 1] = l;
      }
      tc_fence_before();
      mbar_arrive(&sh.o_empty);
    }
  }

  // ---- teardown: drain this CTA's tensor-core work, then free tensor memory
  if (warp == 1) {
    __syncwarp();
    umma_commit(&sh.drain);  // arrives once every MMA issued by lane 0 has completed
    mbar_wait(&sh.drain, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(S::TMEM_COLS) : "memory");
  }
}

// ------------------------------------------------------------------ host side

int cascade_supported(int group, int head_dim) {
  return (head_dim == 64 || head_dim == 128 || head_dim == 256) && group >= 1 && group <= CS_M;
}

size_t cascade_partials_bytes(int num_seqs, int num_q_heads, int head_dim) {
  // per (sequence, query head): the prefix slices, then one slot for the decode kernel's own partial
  return static_cast<size_t>(num_seqs) * num_q_heads * (CASCADE_SPLITS + 1) * cascade_record_floats(head_dim) *
         sizeof(float);
}

template <int D>
static int launch_cascade_t(const CascadeParams& p, const void* q, const void* k_cache, const void* v_cache,
                            int total_q_tokens, cudaStream_t stream, int num_sms) {
  using S = CascadeShape<D>;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return PA_ERR_CUDA;
  const int tokm = cascade_tokm(p.group);
  CUtensorMap tq, tk, tv;
  {  // q [Tq, Hq, D] as (D, Hq, Tq); box = 64 columns x G heads x tokm sequences
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(p.num_q_heads),
                                static_cast<cuuint64_t>(total_q_tokens)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(p.num_q_heads) * D * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(p.group), static_cast<cuuint32_t>(tokm)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (fn(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cu_fail(CUDA_ERROR_INVALID_VALUE, "cuTensorMapEncodeTiled");
  }
  for (int which = 0; which < 2; ++which) {  // caches as (D, bs, Hkv, NB); box = 64 columns x 16 rows
    const cuuint64_t row = static_cast<cuuint64_t>(D) * 2;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(p.block_size),
                                static_cast<cuuint64_t>(p.num_kv_heads), static_cast<cuuint64_t>(p.num_blocks)};
    const cuuint64_t strides[3] = {row, row * p.block_size, row * p.block_size * p.num_kv_heads};
    const cuuint32_t box[4] = {64, 16, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (fn(which ? &tv : &tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(which ? v_cache : k_cache),
           dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cu_fail(CUDA_ERROR_INVALID_VALUE, "cuTensorMapEncodeTiled");
  }
  auto kern = cascade_kernel<D>;
  const int smem = S::SMEM_TOTAL + 1024;
  static PerDevice configured;
  int done = 0;
  const int rc_setup = per_device(
      configured,
      [&](int) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        return e == cudaSuccess ? 1 : cuda_fail(e, "cudaFuncSetAttribute");
      },
      &done);
  if (rc_setup != PA_OK) return rc_setup;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms));  // persistent: the item count is known on the device only
  cfg.blockDim = dim3(CS_THREADS);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return check_launch(cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p), "cascade_kernel launch");
}

int launch_cascade(const CascadeParams& p, const void* q, const void* k_cache, const void* v_cache,
                   int total_q_tokens, int head_dim, cudaStream_t stream, int num_sms) {
  switch (head_dim) {
    case 64: return launch_cascade_t<64>(p, q, k_cache, v_cache, total_q_tokens, stream, num_sms);
    case 128: return launch_cascade_t<128>(p, q, k_cache, v_cache, total_q_tokens, stream, num_sms);
    case 256: return launch_cascade_t<256>(p, q, k_cache, v_cache, total_q_tokens, stream, num_sms);
    default: return PA_ERR_UNSUPPORTED;
  }
}

}  // namespace pa
