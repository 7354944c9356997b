// pa_chunk.cu -- causal attention of prefill chunks over the paged KV cache on
// the 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// What it computes ("vLLM serving internals", AI Engineering from Scratch,
// Phase 17 / 04, "Chunked prefill protects the TTFT tail"; "Inference
// optimization", Phase 10 / 12, "Build it -- Step 2"): the qlen query rows of
// a chunk are the last qlen positions of the sequence; row i (position
// p0 + i, p0 = context_len - qlen) attends to keys 0 .. p0 + i, gathered
// through the block table.
//
// How (B200):
//  * M-tile = 128 query rows: TOK consecutive tokens x the G query heads of
//    one KV head (GQA packing: every K/V tile feeds all G heads); TOK = 128/G
//    for G = 1, 2, 4, 8, 16, and 20 or 10 tokens (120 rows, 8 of padding) for
//    G = 6 or 12.  A work item
//    is a PAIR of consecutive M-tiles (A and B) of one KV head: both multiply
//    the same K/V tiles, so each tile crosses L2 -> shared memory once per
//    256 query rows.  Head dim D = 128 or 64: a row is D/64 panels of 64
//    columns.  Q comes in with one 3-D TMA box per panel and M-tile (128 rows
//    x 128 bytes, 128-byte swizzle) -- a K-major UMMA operand as it lands.
//  * N-tile = 128 keys: 128/block_size blocks, each fetched with 16-row TMA
//    boxes straight into K-major SW128 panels (K for S = Q K^T) and the same
//    panels serve as the MN-major B operand of O += P V.
//  * Warp roles (12 warps, 3 warpgroups): warp 0 issues TMA; warp 1 allocates
//    tensor memory and issues tcgen05.mma (the warp converged, lane 0 under a
//    predicate: a branch that only lane 0 takes makes each issue cost 2-3
//    times the MMA's own 64 cycles); warpgroup 1 runs
//    the softmax of M-tile A, warpgroup 2 that of M-tile B (thread = TMEM lane
//    = query row).  Warpgroup 0 gives registers to the two softmax
//    warpgroups (setmaxnreg).  Tensor memory: S_A, S_B (128 fp32 columns
//    each; P overwrites the first 64 columns of its S as bf16 pairs and is
//    the A operand of P V straight from tensor memory) and O_A, O_B (D
//    columns each, 128 apart).  The MMA issue order QK_A(j), QK_B(j), PV_A(j), QK_A(j+1),
//    PV_B(j), QK_B(j+1), ... lets the tensor cores work on one M-tile while the
//    softmax of the other runs.
//  * Softmax: row max and exp2 on the thread's own row (no shuffles), causal
//    mask on diagonal tiles only, O is rescaled in TMEM only when the running
//    maximum rises by more than 2^8 (between rescales the stale maximum is an
//    exact reference point).  Key rows past the context are zeroed in V
//    before P V.
//  * Work split: with no more items than CTAs, one whole item per CTA (the
//    CTAs of a KV head then read its key tiles in step, from L2).  Otherwise
//    stream-K: the batch's (item, 128-key tile) units, in item order, are cut
//    into one equal contiguous range per CTA, so every CTA gets the same
//    number of tiles whatever the item count.  An item cut by a range
//    boundary leaves unnormalised (O, m, l) pieces, one per CTA that touched
//    it, in that CTA's two piece slots; per (item, row) an atomic count tells
//    the thread that lands the row's last piece to merge the row's pieces in
//    CTA order, write it and put the count back to zero.
//  * Beside the decode kernel: launched after it on part of the GPU, the
//    kernel takes the other SMs while the decode rows stream; it then waits
//    for that grid at its end rather than its start (the decode kernel
//    releases it only after the cache append before both has completed).
//  * Every wait is bounded; on a timeout the CTA raises PA_ERR_TIMEOUT, stops
//    all roles through a shared abort flag, drains its tensor-core work and
//    frees its tensor memory.
#include <cuda.h>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_umma.cuh"

namespace pa {

namespace {

constexpr int CH_THREADS = 384;
constexpr int CH_D_MAX = 128;              // head_dim 64 or 128: one or two 64-column panels
constexpr int CH_M = 128;                   // query rows per M-tile
constexpr int CH_N = 128;                   // keys per N-tile
constexpr int PANEL = CH_M * 128;           // one 128-row x 128-byte swizzled panel (16 KB)
constexpr int KST = 3;                      // K stages (a K tile is free once QK_B of it is done)
constexpr int VST = 2;                      // V stages (a V tile is free once PV_B of it is done)
// Shared memory for head_dim D (D / 64 panels per row block): Q_A, Q_B, then
// the K and V rings.  224 KB at D = 128, 112 KB at D = 64.
template <int D>
struct ChLayout {
  static constexpr int NP = D / 64;              // 64-column panels per row
  static constexpr int Q_BYTES = NP * PANEL;     // one M-tile of Q: [NP panels][128 rows][128 B]
  static constexpr int KV_BYTES = NP * PANEL;    // one K (or V) tile of 128 keys
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = SMEM_Q + 2 * Q_BYTES;
  static constexpr int SMEM_V = SMEM_K + KST * KV_BYTES;
  static constexpr int SMEM_TOTAL = SMEM_V + VST * KV_BYTES;
};
constexpr uint32_t TMEM_COLS = 512;                           // S_A, S_B, O_A, O_B: 128 columns each
// Tokens per M-tile: as many as fit in its 128 rows (TOK x G, one row per
// (token, head)) with a row count that is a multiple of 8 (whole 8-row swizzle
// atoms for the Q box).  128 / G for G a power of two; 20 tokens (120 rows)
// at G = 6 and 10 (120) at G = 12, the last rows then padding.
__host__ __device__ constexpr int chunk_tok(int group) {
  int t = CH_M / group;
  while (t > 1 && (t * group) % 8 != 0) --t;
  return t;
}
constexpr uint32_t TMEM_O = 256;                              // O of M-tile w at TMEM_O + 128 w (D columns)
constexpr float RESCALE_LOG2 = 8.f;                           // rescale O when the max rises by > 2^8
constexpr int SLOT_STRIDE = CH_D_MAX + 4;  // piece slot row: O[D], then m, l (at D), padding
constexpr int MIN_UNITS_PER_CTA = 4;   // key tiles
// What a CTA reads or writes once (Q tiles, piece slots) goes into L2 as
// first to be evicted, ahead of the K/V tiles the other items re-read.
// Register split (setmaxnreg): the launch gives 168 per thread (65,536 / 384,
// rounded down to 8); warpgroup 0 drops to 104, the softmax warpgroups rise to
// 200: 128 x 104 + 256 x 200 = 64,512 = 384 x 168, the launch's total (a
// larger sum would make setmaxnreg.inc wait forever).  Neither side spills.
constexpr int REGS_LAUNCH = 168, REGS_PRODUCER = 104, REGS_SOFTMAX = 200;
static_assert(128 * REGS_PRODUCER + 256 * REGS_SOFTMAX <= CH_THREADS * REGS_LAUNCH, "register split");

struct Item {
  int s;           // sequence
  int q0, qlen;    // its query rows
  int p0, ctx;     // position of its first row, its key count
  int tp, kvh;     // pair of token blocks (2 x 128/G tokens) and KV head
};

struct Shared {
  uint64_t q_full, q_empty, drain;
  uint64_t s_full[2], p_full[2], pv_done[2], o_empty[2];
  uint64_t k_full[KST], k_empty[KST], v_full[VST], v_empty[VST];
  uint32_t tmem_base;
  int abort;
  int merge;        // this CTA landed the last piece of the item being finished
  int units;  // (item, key tile) units of the batch
  int items;  // items with at least one key tile
  int my_lo, my_hi;  // with no more items than CTAs: this CTA's item, as a unit range
};

}  // namespace

// Items = (multi-row sequence, pair of token blocks, KV head), numbered
// sequence by sequence, KV head fastest; an item's units are its key tiles.
// The batch is scanned from global memory by each role (it is small and
// L1-resident).
__device__ __forceinline__ void fill_item(int s, int q0, int qlen, int ctx, int tp, Item& it) {
  it.s = s;
  it.q0 = q0;
  it.qlen = qlen;
  it.ctx = ctx;
  it.p0 = ctx - qlen;
  it.tp = tp;
  it.kvh = 0;
}

// Key tiles an item needs: up to the last position of its pair's last row
// (capped at the context).  M-tile A may see fewer; its extra keys are masked.
__device__ __forceinline__ int item_tiles(const Item& it, int pair_tok) {
  int last = it.p0 + min((it.tp + 1) * pair_tok, it.qlen) - 1;
  if (last >= it.ctx) last = it.ctx - 1;
  return last < 0 ? 0 : last / CH_N + 1;
}

// Total units of the batch.
__device__ __forceinline__ long long chunk_units(const ChunkParams& p, int pair_tok) {
  long long n = 0;
  const int cap = p.max_blocks * p.block_size;
  for (int s = 0; s < p.num_seqs; ++s) {
    const int q0 = __ldg(p.query_start + s), qlen = __ldg(p.query_start + s + 1) - q0;
    if (qlen < p.min_qlen) continue;
    const int ctx = min(__ldg(p.context_lens + s), cap);
    Item it;
    for (int tp = 0; tp * pair_tok < qlen; ++tp) {
      fill_item(s, q0, qlen, ctx, tp, it);
      n += static_cast<long long>(item_tiles(it, pair_tok)) * p.num_kv_heads;
    }
  }
  return n;
}

// The item that holds unit u: the item, its index (for its piece counter),
// its first unit and its tile count.  False if u is past the last unit.
__device__ __forceinline__ bool chunk_unit_item(const ChunkParams& p, int pair_tok, int u, Item& it, int& idx,
                                                int& ubase, int& nt) {
  int base = 0, item_base = 0;
  const int cap = p.max_blocks * p.block_size;
  for (int s = 0; s < p.num_seqs; ++s) {
    const int q0 = __ldg(p.query_start + s), qlen = __ldg(p.query_start + s + 1) - q0;
    if (qlen < p.min_qlen) continue;
    const int ctx = min(__ldg(p.context_lens + s), cap);
    for (int tp = 0; tp * pair_tok < qlen; ++tp) {
      fill_item(s, q0, qlen, ctx, tp, it);
      const int n = item_tiles(it, pair_tok);
      const int units = n * p.num_kv_heads;
      if (u < base + units) {
        const int kvh = (u - base) / n;
        it.kvh = kvh;
        idx = item_base + kvh;
        ubase = base + kvh * n;
        nt = n;
        return true;
      }
      base += units;
      item_base += p.num_kv_heads;
    }
  }
  return false;
}

// Items with at least one key tile, and the unit range of the c-th of them
// (lo = hi = units if there is none).
__device__ __forceinline__ void chunk_items(const ChunkParams& p, int pair_tok, int c, int& count, int& lo, int& hi) {
  count = 0;
  int base = 0;
  lo = hi = -1;
  const int cap = p.max_blocks * p.block_size;
  for (int s = 0; s < p.num_seqs; ++s) {
    const int q0 = __ldg(p.query_start + s), qlen = __ldg(p.query_start + s + 1) - q0;
    if (qlen < p.min_qlen) continue;
    const int ctx = min(__ldg(p.context_lens + s), cap);
    for (int tp = 0; tp * pair_tok < qlen; ++tp) {
      Item it;
      fill_item(s, q0, qlen, ctx, tp, it);
      const int n = item_tiles(it, pair_tok);
      if (n == 0) continue;
      for (int h = 0; h < p.num_kv_heads; ++h, ++count, base += n)
        if (count == c) {
          lo = base;
          hi = base + n;
        }
    }
  }
  if (lo < 0) lo = hi = base;
}

// First unit of CTA c's range, and the CTA whose range holds unit u.
__device__ __forceinline__ int cta_range_start(int units, int c, int ncta) {
  return static_cast<int>(static_cast<long long>(units) * c / ncta);
}
__device__ __forceinline__ int cta_of_unit(int units, int u, int ncta) {
  int c = static_cast<int>(static_cast<long long>(u) * ncta / units);
  while (c + 1 < ncta && cta_range_start(units, c + 1, ncta) <= u) ++c;
  while (c > 0 && cta_range_start(units, c, ncta) > u) --c;
  return c;
}

__device__ __forceinline__ bool ch_wait(Shared& sh, uint64_t* bar, uint32_t phase, int* status) {
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

// A wait taken by a whole warp: every lane polls, and the warp takes one
// answer, so it stays converged for what follows (the MMA warp's predicated
// issue, the softmax warps' warp-collective tensor-memory loads and stores)
// even when the wait runs out in some lanes only.
__device__ __forceinline__ bool ch_wait_warp(Shared& sh, uint64_t* bar, uint32_t phase, int* status) {
  return __all_sync(FULL_MASK, ch_wait(sh, bar, phase, status));
}

// Merge the pieces of one row of a cut item, held by the CTAs c_first ..
// c_last with a non-empty range (slot first_slot for c_first, 0 for the
// others), in CTA order: m = max m_k, out = sum_k 2^(m_k - m) O_k /
// sum_k 2^(m_k - m) l_k; then write the bf16 row (orow == nullptr: a row past
// the chunk, nothing to write).  Kept out of line: the rare path's registers
// stay out of the softmax loop's allocation.
template <int D>
__device__ __noinline__ void merge_row(const float* __restrict__ partials, int units, int ncta, int ubase, int c_first,
                                       int c_last, int first_slot, int wrow, __nv_bfloat16* orow) {
  float mmax = -INFINITY, lsum = 0.f;
  for (int c = c_first; c <= c_last; ++c) {
    if (cta_range_start(units, c + 1, ncta) == cta_range_start(units, c, ncta)) continue;  // no piece
    const int sl = c == c_first ? first_slot : 0;
    const float* src = partials + ((static_cast<long long>(c) * 2 + sl) * 2 * CH_M + wrow) * SLOT_STRIDE;
    mmax = fmaxf(mmax, __ldcg(src + D));
  }
  for (int c = c_first; c <= c_last; ++c) {
    if (cta_range_start(units, c + 1, ncta) == cta_range_start(units, c, ncta)) continue;
    const int sl = c == c_first ? first_slot : 0;
    const float* src = partials + ((static_cast<long long>(c) * 2 + sl) * 2 * CH_M + wrow) * SLOT_STRIDE;
    const float2 ml = __ldcg(reinterpret_cast<const float2*>(src + D));
    lsum += ml.x == -INFINITY ? 0.f : fast_exp2(ml.x - mmax) * ml.y;
  }
  if (!orow) return;
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll 1
  for (int cc = 0; cc < D / 32; ++cc) {
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    for (int c = c_first; c <= c_last; ++c) {
      if (cta_range_start(units, c + 1, ncta) == cta_range_start(units, c, ncta)) continue;
      const int sl = c == c_first ? first_slot : 0;
      const float* src = partials + ((static_cast<long long>(c) * 2 + sl) * 2 * CH_M + wrow) * SLOT_STRIDE;
      const float mk = __ldcg(src + D);
      const float wk = mk == -INFINITY ? 0.f : fast_exp2(mk - mmax);
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float4 v4 = __ldcg(reinterpret_cast<const float4*>(src + cc * 32 + i));
        acc[i] += wk * v4.x;
        acc[i + 1] += wk * v4.y;
        acc[i + 2] += wk * v4.z;
        acc[i + 3] += wk * v4.w;
      }
    }
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
      uint4 u4;
      u4.x = pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
      u4.y = pack_bf16x2(acc[i + 2] * inv, acc[i + 3] * inv);
      u4.z = pack_bf16x2(acc[i + 4] * inv, acc[i + 5] * inv);
      u4.w = pack_bf16x2(acc[i + 6] * inv, acc[i + 7] * inv);
      *reinterpret_cast<uint4*>(orow + cc * 32 + i) = u4;
    }
  }
}

template <int G, int D>
__global__ void __launch_bounds__(CH_THREADS, 1)
    chunk_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                 const __grid_constant__ CUtensorMap tmv, const ChunkParams p) {
  static_assert(D == 64 || D == 128, "head_dim");
  using L = ChLayout<D>;
  constexpr int TOK = chunk_tok(G);  // tokens per M-tile
  constexpr int QROWS = TOK * G;     // its rows that hold a (token, head); the rest are padding
  constexpr int PAIR = 2 * TOK;      // tokens per item
  extern __shared__ uint8_t smem_raw[];
  __shared__ Shared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sh.q_full, 1);
    mbar_init(&sh.q_empty, 1);
    mbar_init(&sh.drain, 1);
    for (int w = 0; w < 2; ++w) {
      mbar_init(&sh.s_full[w], 1);
      mbar_init(&sh.p_full[w], 128);
      mbar_init(&sh.pv_done[w], 1);
      mbar_init(&sh.o_empty[w], 128);
    }
    for (int b = 0; b < KST; ++b) {
      mbar_init(&sh.k_full[b], 1);
      mbar_init(&sh.k_empty[b], 1);
    }
    for (int b = 0; b < VST; ++b) {
      mbar_init(&sh.v_full[b], 1);
      mbar_init(&sh.v_empty[b], 1);
    }
    sh.abort = 0;
    const long long u_all = chunk_units(p, PAIR);
    if (u_all > 0x7fffffffLL) set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));  // far beyond any real batch
    sh.units = u_all > 0x7fffffffLL ? 0 : static_cast<int>(u_all);
    // with no more items than CTAs every CTA takes one whole item: no item is
    // cut, and the CTAs of a KV head walk its key tiles in step (each tile
    // crosses HBM once and is then read from L2 by the others)
    chunk_items(p, PAIR, static_cast<int>(blockIdx.x), sh.items, sh.my_lo, sh.my_hi);
    fence_mbar_init();
  }
  if (warp == 1) {  // tensor memory: S_A, S_B, O_A, O_B
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh.tmem_base)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  // the cache may still be being appended by the kernel before this one
  // (beside the decode kernel: that kernel released this one after it had
  // waited for the append itself, and this one waits for it at the end)
  if (!p.dep_at_end) grid_dependency_wait();

  // this CTA's contiguous range [ua, ub) of the batch's (item, key tile) units
  // (at least MIN_UNITS_PER_CTA units per CTA: a small batch on fewer CTAs,
  // so that its items are not cut into one-tile pieces; the others idle)
  const int units = sh.units;
  const bool whole_items = sh.items <= static_cast<int>(gridDim.x);
  const int ncta = max(1, min(static_cast<int>(gridDim.x), units / MIN_UNITS_PER_CTA));
  const int cta = static_cast<int>(blockIdx.x);
  const int ua = whole_items ? sh.my_lo : cta < ncta ? cta_range_start(units, cta, ncta) : units;
  const int ub = whole_items ? sh.my_hi : cta < ncta ? cta_range_start(units, cta + 1, ncta) : units;
  if (warp < 4) {
    // ================================================================ warpgroup 0
    regs_dec<REGS_PRODUCER>();
    if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmq);
      prefetch_tmap(&tmk);
      prefetch_tmap(&tmv);
    }
    const uint64_t pol = policy_evict_last();  // a chunk's K/V is re-read by every item of the chunk
    uint32_t items = 0, tcount = 0;  // tiles issued over all items (stage and phase bookkeeping)
    for (int u = ua; u < ub && !sh.abort; ++items) {
      Item it;
      int idx, ubase, nt;
      if (!chunk_unit_item(p, PAIR, u, it, idx, ubase, nt)) break;
      // this CTA's piece of the item: key tiles j0 .. j1 - 1
      const int j0 = u - ubase;
      const int j1 = ub - ubase < nt ? ub - ubase : nt;
      u = ubase + j1;
      const int nblk_ctx = (it.ctx + p.block_size - 1) / p.block_size;
      const int32_t* table = p.block_tables + static_cast<long long>(it.s) * p.max_blocks;
      // lane b < 8 owns the b-th 16-key group of a tile: block id and row offset in the block
      auto tile_ids = [&](int j, int& blk, int& y) {
        blk = -1;
        y = 0;
        if (lane < CH_N / 16 && j < nt) {
          const int key0 = j * CH_N + lane * 16;
          const int lb = key0 / p.block_size;
          y = key0 - lb * p.block_size;
          if (lb < nblk_ctx) blk = __ldg(table + lb);
        }
      };
      int blk_cur, y_cur, blk_prev = -1, y_prev = 0, blk_next, y_next;
      tile_ids(j0, blk_cur, y_cur);
      tile_ids(j0 + 1, blk_next, y_next);
      // the previous item's last QK^T has read both Q tiles
      if (items > 0 && !ch_wait(sh, &sh.q_empty, (items - 1) & 1, p.status)) break;
      if (lane == 0) {
        const int t0 = it.q0 + it.tp * PAIR;
        mbar_arrive_expect_tx(&sh.q_full, 2 * L::NP * QROWS * 128);  // the boxes' bytes
        const uint64_t qpol = policy_evict_first();
#pragma unroll
        for (int pn = 0; pn < L::NP; ++pn) {  // panel pn: head-dim columns 64 pn .. 64 pn + 63
          tma_load_3d_hint(smem + L::SMEM_Q + pn * PANEL, &tmq, &sh.q_full, 64 * pn, it.kvh * G, t0, qpol);
          tma_load_3d_hint(smem + L::SMEM_Q + L::Q_BYTES + pn * PANEL, &tmq, &sh.q_full, 64 * pn, it.kvh * G,
                           t0 + TOK, qpol);
        }
      }
      auto load_tile = [&](const CUtensorMap* tm, uint64_t* bars_full, uint64_t* bars_empty, int nst, int base_off,
                           uint32_t t, int blk, int y) -> bool {
        const int st = t % nst;
        const uint32_t use = t / nst;  // earlier fills of this stage
        if (use > 0 && !ch_wait(sh, &bars_empty[st], (use - 1) & 1, p.status)) return false;
        if (lane == 0) mbar_arrive_expect_tx(&bars_full[st], L::KV_BYTES);
        __syncwarp();
        if (lane < CH_N / 16) {  // 16-row boxes (one 64-column panel, 16 keys) -> rows 16*lane.. of every panel
          if (blk >= p.num_blocks) set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
          uint8_t* dst = smem + base_off + st * L::KV_BYTES + lane * 2048;
#pragma unroll
          for (int pn = 0; pn < L::NP; ++pn) tma_load_4d(dst + pn * PANEL, tm, &bars_full[st], 64 * pn, y, it.kvh, blk, pol);
        }
        return true;
      };
      bool ok = true;
      for (int j = j0; ok && j < j1; ++j) {
        ok = load_tile(&tmk, sh.k_full, sh.k_empty, KST, L::SMEM_K, tcount + (j - j0), blk_cur, y_cur);
        if (ok && j > j0)
          ok = load_tile(&tmv, sh.v_full, sh.v_empty, VST, L::SMEM_V, tcount + (j - j0) - 1, blk_prev, y_prev);
        blk_prev = blk_cur;
        y_prev = y_cur;
        blk_cur = blk_next;
        y_cur = y_next;
        tile_ids(j + 2, blk_next, y_next);  // one tile of lead for the block-table reads
      }
      if (ok && j1 > j0)
        ok = load_tile(&tmv, sh.v_full, sh.v_empty, VST, L::SMEM_V, tcount + (j1 - j0) - 1, blk_prev, y_prev);
      tcount += j1 - j0;
      if (!ok) break;
    }
    if (sh.abort) {  // let this CTA's copies still in flight land before its shared memory goes away
      for (int st = 0; st < KST; ++st) {
        const uint32_t uses = tcount / KST + (static_cast<uint32_t>(st) < tcount % KST ? 1u : 0u);
        if (uses > 0) mbar_wait(&sh.k_full[st], (uses - 1) & 1);
      }
      for (int st = 0; st < VST; ++st) {
        const uint32_t uses = tcount / VST + (static_cast<uint32_t>(st) < tcount % VST ? 1u : 0u);
        if (uses > 0) mbar_wait(&sh.v_full[st], (uses - 1) & 1);
      }
      if (items > 0) mbar_wait(&sh.q_full, (items - 1) & 1);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    const uint32_t idesc_qk = umma_idesc(CH_M, CH_N, 0, 0);
    const uint32_t idesc_pv = umma_idesc(CH_M, D, 0, 1);
    const uint32_t sq = smem_u32(smem + L::SMEM_Q);
    uint32_t q_phase = 0, p_phase[2] = {0, 0}, o_phase = 0, kv_count = 0;
    uint32_t pv_commits[2] = {0, 0};  // completions committed to pv_done[w] so far
    bool first_item = true;
    for (int u = ua; u < ub && !sh.abort;) {
      Item it;
      int idx, ubase, nt;
      if (!chunk_unit_item(p, PAIR, u, it, idx, ubase, nt)) break;
      // this CTA's piece of the item: key tiles j0 .. j1 - 1
      const int j0 = u - ubase;
      const int j1 = ub - ubase < nt ? ub - ubase : nt;
      u = ubase + j1;
      if (!ch_wait_warp(sh, &sh.q_full, q_phase, p.status)) break;
      q_phase ^= 1;
      if (!first_item) {  // both epilogues of the previous item have read O
        if (!ch_wait_warp(sh, &sh.o_empty[0], o_phase, p.status) ||
            !ch_wait_warp(sh, &sh.o_empty[1], o_phase, p.status))
          break;
        o_phase ^= 1;
      }
      first_item = false;
      if (j1 <= j0) {  // nothing to multiply: Q is free, and each epilogue gets its one P V completion
        umma_commit(&sh.q_empty);
        umma_commit(&sh.pv_done[0]);
        umma_commit(&sh.pv_done[1]);
        ++pv_commits[0];
        ++pv_commits[1];
        continue;
      }
      // S_w(j) = Q_w K(j)^T.  S_w last held P_w(j - 1), the A operand of
      // P V_w(j - 1): wait until that MMA has completed before overwriting it
      // (for j = 0, the previous item's epilogue already waited for its last P V).
      auto qk = [&](int w, int j) -> bool {
        const uint32_t t = kv_count + (j - j0);  // tiles this CTA has taken so far
        const int stage = t % KST;
        if (w == 0 && !ch_wait_warp(sh, &sh.k_full[stage], (t / KST) & 1, p.status)) return false;
        if (j > j0 && !ch_wait_warp(sh, &sh.pv_done[w], (pv_commits[w] - 1) & 1, p.status)) return false;
        tc_fence_after();
        const uint32_t sk = smem_u32(smem + L::SMEM_K + stage * L::KV_BYTES);
        const uint32_t qw = sq + w * L::Q_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * PANEL + (kk & 3) * 32;
          umma_f16(tmem + w * CH_N, umma_desc(qw + off, 16, 1024), umma_desc(sk + off, 16, 1024), idesc_qk, kk > 0);
        }
        umma_commit(&sh.s_full[w]);
        if (w == 1) {
          umma_commit(&sh.k_empty[stage]);
          if (j == j1 - 1) umma_commit(&sh.q_empty);
        }
        return true;
      };
      // O_w += P_w(j) V(j), P_w(j) in the first 64 columns of S_w
      auto pv = [&](int w, int j) -> bool {
        if (!ch_wait_warp(sh, &sh.p_full[w], p_phase[w], p.status)) return false;
        p_phase[w] ^= 1;
        const uint32_t t = kv_count + (j - j0);
        const int stage = t % VST;
        if (w == 0 && !ch_wait_warp(sh, &sh.v_full[stage], (t / VST) & 1, p.status)) return false;
        tc_fence_after();
        const uint32_t sv = smem_u32(smem + L::SMEM_V + stage * L::KV_BYTES);
        const uint32_t pt = tmem + w * CH_N;
#pragma unroll
        for (int kk = 0; kk < CH_N / 16; ++kk)  // keys 16kk.. = P columns 8kk..; V rows 16kk.., both panels
          umma_f16_ts(tmem + TMEM_O + w * CH_N, pt + 8 * kk, umma_desc(sv + kk * 16 * 128, PANEL, 1024), idesc_pv,
                      (j > j0 || kk > 0) ? 1u : 0u);
        umma_commit(&sh.pv_done[w]);
        if (w == 1) umma_commit(&sh.v_empty[stage]);
        ++pv_commits[w];
        return true;
      };
      bool ok = qk(0, j0) && qk(1, j0);
      for (int j = j0 + 1; ok && j < j1; ++j) ok = pv(0, j - 1) && qk(0, j) && pv(1, j - 1) && qk(1, j);
      if (ok) ok = pv(0, j1 - 1) && pv(1, j1 - 1);
      kv_count += j1 - j0;
      if (!ok) break;
    }
    }
  } else {
    // ================================================================ softmax warpgroups
    regs_inc<REGS_SOFTMAX>();
    const int w = (warp >> 2) - 1;        // 0: M-tile A, 1: M-tile B
    const int quad = warp & 3;            // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;     // query row of the M-tile = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_col = tmem + lane_addr + w * CH_N, o_col = tmem + lane_addr + TMEM_O + w * CH_N;
    const int tok_in_tile = row / G, head_in_group = row % G;
    // kv_count: key tiles of earlier items (V stages); pv_count: completions
    // of pv_done[w] so far (one per tile, one for an item without tiles)
    uint32_t s_phase = 0, kv_count = 0, pv_count = 0;
    for (int u = ua; u < ub && !sh.abort;) {
      Item it;
      int idx, ubase, nt;
      if (!chunk_unit_item(p, PAIR, u, it, idx, ubase, nt)) break;
      // this CTA's piece of the item: key tiles j0 .. j1 - 1
      const int j0 = u - ubase;
      const int j1 = ub - ubase < nt ? ub - ubase : nt;
      u = ubase + j1;
      const int tok = it.tp * PAIR + w * TOK + tok_in_tile;  // row's token within the chunk
      const int last_key = it.p0 + tok;                       // causal limit (inclusive)
      const bool row_valid = row < QROWS && tok < it.qlen && last_key >= 0;
      const int tile_last = it.p0 + it.tp * PAIR + w * TOK;   // first row of this M-tile: keys beyond it are
                                                              // masked for some row of the tile

      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = j0; j < j1 && ok; ++j) {
        if (!(ok = ch_wait_warp(sh, &sh.s_full[w], s_phase, p.status))) break;
        s_phase ^= 1;
        tc_fence_after();
        float s[CH_N];
#pragma unroll
        for (int c = 0; c < CH_N / 32; ++c) {
          float v[32];
          tmem_ld32(s_col + c * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = v[i];
        }
        tmem_wait_ld();

        const int key0 = j * CH_N;
        const bool diag = key0 + CH_N - 1 > tile_last;  // some row of the tile stops inside (or before) it
        const float cs = p.scale_log2;
        // Off the diagonal every key is visible: take the max of the raw scores
        // and fold the scale into one FFMA per element below.  On a diagonal
        // tile scale first, then mask (the scale may be zero).
        float mx;
        {
          float m8[8];
          if (diag) {
#pragma unroll
            for (int i = 0; i < CH_N; ++i) {
              const float x = s[i] * cs;
              s[i] = key0 + i > last_key ? -INFINITY : x;
            }
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = s[k];
          if (diag || cs >= 0.f) {
#pragma unroll
            for (int i = 8; i < CH_N; i += 8)
#pragma unroll
              for (int k = 0; k < 8; ++k) m8[k] = fmaxf(m8[k], s[i + k]);
            mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
          } else {  // raw scores and a negative scale: the smallest raw score scales to the largest
#pragma unroll
            for (int i = 8; i < CH_N; i += 8)
#pragma unroll
              for (int k = 0; k < 8; ++k) m8[k] = fminf(m8[k], s[i + k]);
            mx = fminf(fminf(fminf(m8[0], m8[1]), fminf(m8[2], m8[3])), fminf(fminf(m8[4], m8[5]), fminf(m8[6], m8[7])));
          }
          if (!diag) mx *= cs;
        }
        const bool rescale = mx > m_ref + RESCALE_LOG2 || m_ref == -INFINITY;
        const float m_new = rescale ? fmaxf(mx, m_ref) : m_ref;
        // P in bf16 pairs (keys 2c, 2c + 1 in column c), straight into S_w
        const float neg_m = (m_new == -INFINITY) ? 0.f : -m_new;  // a row with no key yet: P = 0, not NaN
        float l8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < CH_N / 64; ++c) {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float x0 = s[64 * c + 2 * i], x1 = s[64 * c + 2 * i + 1];
            const float a = fast_exp2(diag ? x0 + neg_m : fmaf(x0, cs, neg_m));
            const float b = fast_exp2(diag ? x1 + neg_m : fmaf(x1, cs, neg_m));
            l8[i & 7] += a + b;
            pk[i] = pack_bf16x2(a, b);
          }
          tmem_st32u(s_col + 32 * c, pk);
        }
        const bool resc = rescale && m_ref != -INFINITY;
        const float alpha = resc ? fast_exp2(m_ref - m_new) : 1.f;
        l = l * alpha + (((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7])));
        m_ref = m_new;
        // O holds tiles 0..j-1: wait for P V_w(j - 1), then scale O in tensor
        // memory.  tcgen05.ld/st are warp-collective, so the whole warp takes
        // this branch when any of its rows rescales (the others scale by 1).
        if (j > j0 && __any_sync(FULL_MASK, resc)) {
          // pv_done[w] completes once per tile; P V_w(j) cannot have completed
          // (it waits for this thread's P), so the parity names the phase
          if (!(ok = ch_wait_warp(sh, &sh.pv_done[w], (pv_count + (j - j0) - 1) & 1, p.status))) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float v[32];
            tmem_ld32(o_col + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= alpha;
            tmem_st32(o_col + c * 32, v);
          }
        }
        tmem_wait_st();
        // keys past the context may hold anything (even NaN): zero their V rows
        // (M-tile A's warpgroup does it; P V_B(j) is issued after P V_A(j))
        const int valid_keys = it.ctx - key0;
        if (w == 0 && valid_keys < CH_N) {
          const uint32_t t = kv_count + (j - j0);
          const int stage = t % VST;
          if (!(ok = ch_wait_warp(sh, &sh.v_full[stage], (t / VST) & 1, p.status))) break;
          uint8_t* vst = smem + L::SMEM_V + stage * L::KV_BYTES;
          constexpr int CPR = D / 8;  // 16-byte chunks of a key row, over all panels
          const int nz = (CH_N - max(valid_keys, 0)) * CPR;
          for (int k = threadIdx.x - 128; k < nz; k += 128) {
            const int r = max(valid_keys, 0) + k / CPR, rest = k % CPR;
            *reinterpret_cast<uint4*>(vst + (rest >> 3) * PANEL + r * 128 + (rest & 7) * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        mbar_arrive(&sh.p_full[w]);
      }
      kv_count += j1 - j0;
      pv_count += j1 > j0 ? j1 - j0 : 1;
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 -> out (after the item's last pv_done completion)
      if (!ch_wait_warp(sh, &sh.pv_done[w], (pv_count - 1) & 1, p.status)) break;
      tc_fence_after();
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) +
                            (static_cast<long long>(it.q0 + tok) * p.num_q_heads + it.kvh * G + head_in_group) * D;
      if (j0 == 0 && j1 == nt) {  // the whole item: O / l -> bf16 -> out
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float v[32];
          if (nt > 0) {
            tmem_ld32(o_col + c * 32, v);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
          }
          if (row_valid) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 u4;
              u4.x = pack_bf16x2(v[i] * inv, v[i + 1] * inv);
              u4.y = pack_bf16x2(v[i + 2] * inv, v[i + 3] * inv);
              u4.z = pack_bf16x2(v[i + 4] * inv, v[i + 5] * inv);
              u4.w = pack_bf16x2(v[i + 6] * inv, v[i + 7] * inv);
              *reinterpret_cast<uint4*>(orow + c * 32 + i) = u4;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&sh.o_empty[w]);
        continue;
      }
      // ---- a piece of a cut item: the unnormalised (O, m, l) of this row go
      // to this CTA's slot (0: the first piece of its range, 1: the last).
      // The CTAs c_first .. c_last with a non-empty range hold the item's
      // pieces (with more CTAs than units some ranges are empty); c_first's is
      // the last piece of its range (slot 1) unless its range starts with the
      // item, every later one the first piece of its range (slot 0).
      const int my_slot = (ubase + j0 == ua) ? 0 : 1;
      const int wrow = w * CH_M + row;  // row of the item (both M-tiles)
      float* dst = p.partials + ((static_cast<long long>(cta) * 2 + my_slot) * 2 * CH_M + wrow) * SLOT_STRIDE;
      const uint64_t spol = policy_evict_first();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tmem_ld32(o_col + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          st_global_hint(reinterpret_cast<float4*>(dst + c * 32 + i), make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]),
                         spol);
      }
      __stcg(reinterpret_cast<float2*>(dst + D), make_float2(m_ref, l));
      tc_fence_before();
      mbar_arrive(&sh.o_empty[w]);  // O has been read
      // One count per (item, row): the thread that lands a row's last piece
      // merges that row, with no wait on any other thread.
      __threadfence();
      const int c_first = cta_of_unit(units, ubase, ncta), c_last = cta_of_unit(units, ubase + nt - 1, ncta);
      const int first_slot = cta_range_start(units, c_first, ncta) == ubase ? 0 : 1;
      int npieces = 0;
      for (int c = c_first; c <= c_last; ++c)
        npieces += cta_range_start(units, c + 1, ncta) > cta_range_start(units, c, ncta);
      int* const cnt = p.counters + static_cast<long long>(idx) * (2 * CH_M) + wrow;
      if (atomicAdd(cnt, 1) != npieces - 1) continue;
      *cnt = 0;  // every piece of this row has arrived: back to zero for the next call
      __threadfence();
      merge_row<D>(p.partials, units, ncta, ubase, c_first, c_last, first_slot, wrow, row_valid ? orow : nullptr);
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
  // beside the decode kernel: this grid completes only after that one has, so
  // the stream's later work is ordered after both
  if (p.dep_at_end) grid_dependency_wait();
}

// ------------------------------------------------------------------ host side

int chunk_supported(int group, int head_dim) {
  return (head_dim == 64 || head_dim == 128) &&
         (group == 1 || group == 2 || group == 4 || group == 6 || group == 8 || group == 12 || group == 16);
}

// q [Tq, Hq, D] bf16 as a 3-D tensor (D, Hq, Tq); box = 64 columns x G heads x chunk_tok(G) tokens.
static int encode_q_tmap(CUtensorMap* map, const void* q, int total_q_tokens, int num_q_heads, int group,
                         int head_dim, EncodeTiledFn fn) {
  const cuuint64_t d = static_cast<cuuint64_t>(head_dim);
  const cuuint64_t dims[3] = {d, static_cast<cuuint64_t>(num_q_heads), static_cast<cuuint64_t>(total_q_tokens)};
  const cuuint64_t strides[2] = {d * 2, static_cast<cuuint64_t>(num_q_heads) * d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(chunk_tok(group))};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : cu_fail(r, "cuTensorMapEncodeTiled");
}

// [num_blocks, Hkv, block_size, D] as a 4-D tensor; box = 64 columns x 16 rows of one (block, head).
int encode_kv16_tmap(CUtensorMap* map, const void* cache, int num_blocks, int num_kv_heads, int block_size,
                     int head_dim, EncodeTiledFn fn) {
  const cuuint64_t row = static_cast<cuuint64_t>(head_dim) * 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(block_size),
                              static_cast<cuuint64_t>(num_kv_heads),
                              static_cast<cuuint64_t>(num_blocks)};
  const cuuint64_t strides[3] = {row, row * block_size, row * block_size * num_kv_heads};
  const cuuint32_t box[4] = {64, 16, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(cache), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : cu_fail(r, "cuTensorMapEncodeTiled");
}

template <int G, int D>
static int launch_chunk_t(const ChunkParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          cudaStream_t stream, int num_sms, int ctas) {
  auto kern = chunk_kernel<G, D>;
  const int smem = ChLayout<D>::SMEM_TOTAL + 1024;
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
  const int grid = ctas > 0 && ctas < num_sms ? ctas : num_sms;  // one CTA per SM, one unit range each
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(CH_THREADS);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return check_launch(cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p), "chunk_kernel launch");
}

// Items of a batch: pairs of M-tiles (2 chunk_tok(G) tokens) of each multi-row
// sequence, times the KV heads; at most (rows / (2 chunk_tok(G)) + sequences)
// * Hkv.
static size_t chunk_max_items(int num_query_tokens, int num_seqs_bound, int num_kv_heads, int group) {
  return (static_cast<size_t>(num_query_tokens) / (2 * chunk_tok(group)) + static_cast<size_t>(num_seqs_bound)) *
         static_cast<size_t>(num_kv_heads);
}

static size_t round256_c(size_t n) { return (n + 255) / 256 * 256; }

size_t chunk_workspace_bytes(int num_query_tokens, int num_seqs_bound, int num_kv_heads, int group, int num_sms) {
  const size_t counters = chunk_max_items(num_query_tokens, num_seqs_bound, num_kv_heads, group) * 2 * CH_M * sizeof(int);
  const size_t slots = static_cast<size_t>(num_sms) * 2 * 2 * CH_M * SLOT_STRIDE * sizeof(float);
  return round256_c(counters) + slots;
}

void chunk_workspace_layout(void* ws, int num_query_tokens, int num_seqs_bound, int num_kv_heads, int group,
                            int num_sms, ChunkParams* p) {
  (void)num_sms;
  uint8_t* b = static_cast<uint8_t*>(ws);
  p->counters = reinterpret_cast<int*>(b);
  b += round256_c(chunk_max_items(num_query_tokens, num_seqs_bound, num_kv_heads, group) * 2 * CH_M * sizeof(int));
  p->partials = reinterpret_cast<float*>(b);
}

int launch_chunk(const ChunkParams& p, const void* q, const void* k_cache, const void* v_cache, int total_q_tokens,
                 cudaStream_t stream, int num_sms, int ctas) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return PA_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  int rc;
  if (!chunk_supported(p.group, p.head_dim)) return PA_ERR_UNSUPPORTED;
  if ((rc = encode_q_tmap(&tq, q, total_q_tokens, p.num_q_heads, p.group, p.head_dim, fn)) != PA_OK) return rc;
  if ((rc = encode_kv16_tmap(&tk, k_cache, p.num_blocks, p.num_kv_heads, p.block_size, p.head_dim, fn)) != PA_OK)
    return rc;
  if ((rc = encode_kv16_tmap(&tv, v_cache, p.num_blocks, p.num_kv_heads, p.block_size, p.head_dim, fn)) != PA_OK)
    return rc;
  const bool d64 = p.head_dim == 64;
  switch (p.group) {
    case 1: return d64 ? launch_chunk_t<1, 64>(p, tq, tk, tv, stream, num_sms, ctas)
                       : launch_chunk_t<1, 128>(p, tq, tk, tv, stream, num_sms, ctas);
    case 2: return d64 ? launch_chunk_t<2, 64>(p, tq, tk, tv, stream, num_sms, ctas)
                       : launch_chunk_t<2, 128>(p, tq, tk, tv, stream, num_sms, ctas);
    case 4: return d64 ? launch_chunk_t<4, 64>(p, tq, tk, tv, stream, num_sms, ctas)
                       : launch_chunk_t<4, 128>(p, tq, tk, tv, stream, num_sms, ctas);
    case 6: return d64 ? launch_chunk_t<6, 64>(p, tq, tk, tv, stream, num_sms, ctas)
                       : launch_chunk_t<6, 128>(p, tq, tk, tv, stream, num_sms, ctas);
    case 8: return d64 ? launch_chunk_t<8, 64>(p, tq, tk, tv, stream, num_sms, ctas)
                       : launch_chunk_t<8, 128>(p, tq, tk, tv, stream, num_sms, ctas);
    case 12: return d64 ? launch_chunk_t<12, 64>(p, tq, tk, tv, stream, num_sms, ctas)
                        : launch_chunk_t<12, 128>(p, tq, tk, tv, stream, num_sms, ctas);
    case 16: return d64 ? launch_chunk_t<16, 64>(p, tq, tk, tv, stream, num_sms, ctas)
                        : launch_chunk_t<16, 128>(p, tq, tk, tv, stream, num_sms, ctas);
    default: return PA_ERR_UNSUPPORTED;
  }
}

}  // namespace pa
