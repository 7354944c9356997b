// pa_verify.cu -- attention of short multi-row queries (2 .. 64/G rows per
// sequence, as when a target model checks draft tokens) over the paged KV
// cache, on the 5th-generation tensor cores with the keys in M.
//
// What it computes ("Inference optimization", AI Engineering from Scratch,
// Phase 10 / 12, sections "Speculative decoding", "KV cache" and "Build it --
// Step 2"; "vLLM serving internals", Phase 17 / 04, "PagedAttention as a
// virtual memory system"): row i of sequence s sits at position
// p0 + i, p0 = context_len - qlen, and attends causally to keys 0 .. p0 + i,
// gathered through the block table.
//
// How (B200):
//  * Item = (sequence, KV head).  Its qlen rows x G query heads are the NCOL
//    columns of the item (column = row * G + head; NCOL = 32 or 64, unused
//    columns are computed and dropped).  Per 128-key tile:
//      S^T [128 keys x NCOL] = K_tile . Q^T     A = K tile, B = Q (both K-major,
//                                               128-byte swizzle, landed by TMA)
//    in tensor memory.  One softmax thread per key (TMEM lane): the column
//    maxima come from a warp reduce-scatter and a cross-warp step in shared
//    memory, P goes to shared memory as the K-major A operand of
//      O [NCOL of 128 rows x 128] += P . V_tile  (B = V tile, MN-major)
//    so every K/V byte crosses HBM once for all qlen x G rows, and no M-tile
//    rows are spent on absent tokens of the query block.
//  * Work split: the batch's (item, tile) units in order, cut into equal
//    contiguous ranges, one per CTA (exact to one tile, deterministic).  An
//    item cut by range ends leaves (m, l, O) pieces in per-CTA slots; the CTA
//    that finishes the last piece of an item (a counter per cut item) merges
//    the pieces in CTA order and writes the rows.
//  * Roles (8 warps): warp 0 loads Q and the K tiles, warp 2 the V tiles (each
//    refills its own ring as soon as a stage is free; V, read after the
//    softmax, gets the deeper ring); warp 1 owns tensor memory and issues
//    tcgen05.mma (converged, lane 0 under a predicate) as soon as the inputs
//    of an S or a P V are ready; warps 4-7 run the softmax and the epilogue
//    (thread = TMEM lane).
//    S is double-buffered per tile, P single (written once P V(g - 1) has read
//    it), Q and O per item.  An item's epilogue runs one tile into the next
//    item, when its last P V is known to be complete, so item ends do not
//    stall the pipeline.
//  * O is rescaled only when a column's running maximum rises by more than
//    2^8 (between rescales the stale maximum is an exact reference point).
//  * Every wait is bounded: on a timeout the CTA records PA_ERR_TIMEOUT,
//    stops its roles through a shared flag, lets its copies and MMAs land and
//    frees its tensor memory.
#include <cuda.h>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_umma.cuh"

namespace pa {

namespace {

constexpr int VF_D = 128;                  // head_dim
constexpr int VF_N = 128;                  // keys per tile (the M of S^T)
constexpr int VF_PANEL = VF_N * 128;       // 128 rows x 128 bytes (64 head-dim columns)
constexpr int VF_KV_BYTES = 2 * VF_PANEL;  // one K (or V) tile
constexpr float VF_RESCALE_LOG2 = 8.f;
constexpr uint32_t VF_TMEM_COLS = 512;     // S_0, S_1 at 0 / NCOL; O_0 at 128, O_1 at 256
constexpr uint32_t VF_TMEM_O = 128;
constexpr int VF_SOFTMAX_BAR = 1;          // named barrier of the four softmax warps
constexpr int VF_THREADS = 256;            // warps 0, 2: TMA; 1: MMA; 3: idle; 4-7: softmax and epilogue

template <int NCOL>
struct VfLayout {
  // K is consumed by S one tile ahead of the softmax, V by P V after it: V
  // gets the deeper ring (the bytes in flight set the bandwidth), P a single
  // buffer (the softmax writes P(g) once P V(g - 1) has read P(g - 1))
  static constexpr int KST = 2;                   // K stages
  static constexpr int VST = NCOL == 32 ? 4 : 3;  // V stages
  static constexpr int PP = NCOL * 128;           // one P panel: NCOL rows x 64 keys
  static constexpr int PBUF = 2 * PP;
  static constexpr int QP = NCOL * 128;           // one Q panel: NCOL rows x 64 head-dims
  static constexpr int QBUF = 2 * QP;
  // P first: the P . V MMA (M = 128) reads 128 rows from each P panel, the
  // rows past NCOL land on what follows (unused results, in-bounds reads)
  static constexpr int P_OFF = 0;
  static constexpr int Q_OFF = P_OFF + PBUF;
  static constexpr int K_OFF = Q_OFF + 2 * QBUF;
  static constexpr int V_OFF = K_OFF + KST * VF_KV_BYTES;
  // red[2][4][NCOL] (column maxima of the 4 warps, double-buffered), lred[4][NCOL]
  // (column sums), mv[4][NCOL] (-m per warp), av[4][NCOL] (rescale factors per
  // warp), em[2][NCOL], el[2][NCOL] (m and l of the items whose epilogue may be pending)
  static constexpr int RED_OFF = V_OFF + VST * VF_KV_BYTES;
  static constexpr int RED_FLOATS = 2 * 4 * NCOL + 3 * 4 * NCOL + 4 * NCOL;
  static constexpr int PFX_OFF = RED_OFF + RED_FLOATS * 4;   // long long pfx[VERIFY_SMEM_SEQS + 1]
  static constexpr int BYTES = PFX_OFF + (VERIFY_SMEM_SEQS + 1) * 8;
  static_assert(K_OFF % 1024 == 0 && V_OFF % 1024 == 0 && Q_OFF % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(P_OFF + PBUF + PP + VF_PANEL <= BYTES, "P operand reads stay in shared memory");
  static_assert(BYTES + 1024 <= 227 * 1024, "shared memory");
};

struct VfShared {
  uint64_t q_full[2], q_empty[2], o_empty[2];
  uint64_t s_full[2], s_empty[2], p_full[2], pv_done[2];
  uint64_t k_full[2], k_empty[2], v_full[4], v_empty[4];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int merge;
};

// One item's share of this CTA's unit range.
struct VfItem {
  int s, kvh;
  int q0, qlen, ctx, nt;  // query rows, keys (capped at the table), tiles of the item
  int t0, t1;             // tiles [t0, t1) of the item fall in this CTA's range
  long long base;         // first unit of the item
};

__device__ __forceinline__ bool vf_wait(VfShared& sh, uint64_t* bar, uint32_t phase, int* status) {
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

__device__ __forceinline__ void softmax_bar() {
  asm volatile("bar.sync %0, 128;" ::"n"(VF_SOFTMAX_BAR) : "memory");
}

// Rows of sequence s, and whether this launch (columns in (ncol_lo, ncol_hi]) takes it.
__device__ __forceinline__ bool vf_seq(const VerifyParams& p, int s, int& q0, int& qlen, int& ctx) {
  q0 = __ldg(p.query_start + s);
  qlen = __ldg(p.query_start + s + 1) - q0;
  ctx = __ldg(p.context_lens + s);
  const int cols = qlen * p.group;
  return qlen >= 2 && cols > p.ncol_lo && cols <= p.ncol_hi;
}

__device__ __forceinline__ long long vf_units(const VerifyParams& p, int s) {
  int q0, qlen, ctx;
  if (!vf_seq(p, s, q0, qlen, ctx)) return 0;
  const int cap = p.max_blocks * p.block_size;
  if (ctx > cap) ctx = cap;
  return ctx > 0 ? static_cast<long long>(p.num_kv_heads) * ((ctx + VF_N - 1) / VF_N) : 0;
}

// Fill `it` for the item of sequence s, KV head kvh, whose first unit is `base`.
__device__ __forceinline__ void vf_fill(const VerifyParams& p, int s, int kvh, long long base, long long ua,
                                        long long ub, VfItem& it) {
  int q0, qlen, ctx;
  vf_seq(p, s, q0, qlen, ctx);
  const int cap = p.max_blocks * p.block_size;
  if (ctx > cap) {
    set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
    ctx = cap;
  }
  it.s = s;
  it.kvh = kvh;
  it.q0 = q0;
  it.qlen = qlen;
  it.ctx = ctx;
  it.nt = (ctx + VF_N - 1) / VF_N;
  it.base = base;
  it.t0 = static_cast<int>(ua > base ? ua - base : 0);
  it.t1 = static_cast<int>(ub - base < it.nt ? ub - base : it.nt);
}

// The item holding unit u (u < T), from the shared-memory prefix of unit counts.
__device__ __forceinline__ void vf_seek(const VerifyParams& p, const long long* pfx, long long u, long long ua,
                                        long long ub, VfItem& it) {
  int lo = 0, hi = p.num_seqs - 1;  // last s with pfx[s] <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pfx[mid] <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  // pfx[lo] <= u < pfx[lo + 1]: sequence lo has units
  const long long per = (pfx[lo + 1] - pfx[lo]) / p.num_kv_heads;
  const int kvh = static_cast<int>((u - pfx[lo]) / per);
  vf_fill(p, lo, kvh, pfx[lo] + kvh * per, ua, ub, it);
}

// The item after `it`; false at the end of the range.
__device__ __forceinline__ bool vf_next(const VerifyParams& p, const long long* pfx, long long ua, long long ub,
                                        VfItem& it) {
  const long long next = it.base + it.nt;
  if (next >= ub) return false;
  if (it.kvh + 1 < p.num_kv_heads) {
    vf_fill(p, it.s, it.kvh + 1, next, ua, ub, it);
    return true;
  }
  int s = it.s + 1;
  while (s < p.num_seqs && pfx[s + 1] == pfx[s]) ++s;
  if (s >= p.num_seqs) return false;
  vf_fill(p, s, 0, pfx[s], ua, ub, it);
  return true;
}

// CTA whose range holds unit u: the largest b with floor(T b / n) <= u.
__device__ __forceinline__ int vf_cta_of(long long u, long long T, int n) {
  return static_cast<int>(((u + 1) * n - 1) / T);
}

__device__ __forceinline__ long long vf_range_start(int b, long long T, int n) { return T * b / n; }

// Warp reduce-scatter of 32 values per lane: afterwards lane l holds the
// reduction over the warp of element l.  `op` is max or sum.
template <bool MAX>
__device__ __forceinline__ float vf_reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = up ? v[i] : v[i + w];
      const float keep = up ? v[i + w] : v[i];
      const float r = __shfl_xor_sync(FULL_MASK, send, w);
      v[i] = MAX ? fmaxf(keep, r) : keep + r;
    }
  }
  return v[0];
}

}  // namespace

template <int NCOL>
__global__ void __launch_bounds__(VF_THREADS, 1)
    verify_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const VerifyParams p) {
  using L = VfLayout<NCOL>;
  constexpr int NC32 = NCOL / 32;
  extern __shared__ uint8_t smem_raw[];
  __shared__ VfShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long long* pfx = reinterpret_cast<long long*>(smem + L::PFX_OFF);

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.q_full[b], 1);
      mbar_init(&sh.q_empty[b], 1);
      mbar_init(&sh.o_empty[b], 128);
      mbar_init(&sh.s_full[b], 1);
      mbar_init(&sh.s_empty[b], 128);
      mbar_init(&sh.p_full[b], 128);
      mbar_init(&sh.pv_done[b], 1);
    }
    for (int b = 0; b < L::KST; ++b) {
      mbar_init(&sh.k_full[b], 1);
      mbar_init(&sh.k_empty[b], 1);
    }
    for (int b = 0; b < L::VST; ++b) {
      mbar_init(&sh.v_full[b], 1);
      mbar_init(&sh.v_empty[b], 1);
    }
    mbar_init(&sh.drain, 1);
    sh.abort = 0;
    sh.merge = 0;
    fence_mbar_init();
  }
  // units per sequence, their prefix sums (batch metadata only)
  for (int s = threadIdx.x; s < p.num_seqs; s += VF_THREADS) pfx[s + 1] = vf_units(p, s);
  if (threadIdx.x == 0) pfx[0] = 0;
  __syncthreads();
  if (warp == 0) {
    long long carry = 0;
    for (int b0 = 0; b0 < p.num_seqs; b0 += 32) {
      const int s = b0 + lane;
      long long v = s < p.num_seqs ? pfx[s + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long n = __shfl_up_sync(FULL_MASK, v, o);
        if (lane >= o) v += n;
      }
      if (s < p.num_seqs) pfx[s + 1] = carry + v;
      carry += __shfl_sync(FULL_MASK, v, 31);
    }
  }
  __syncthreads();
  const long long T = pfx[p.num_seqs];
  const int nct = gridDim.x;
  const long long ua = vf_range_start(blockIdx.x, T, nct), ub = vf_range_start(blockIdx.x + 1, T, nct);

  grid_dependency_wait();  // the cache may still be being appended by the kernel before this one
  // rows of taken sequences without a key: zeros (softmax over an empty set)
  for (int s = blockIdx.x; s < p.num_seqs; s += nct) {
    int q0, qlen, ctx;
    if (vf_seq(p, s, q0, qlen, ctx) && ctx <= 0) {
      uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                          static_cast<long long>(q0) * p.num_q_heads * VF_D);
      const int n = qlen * p.num_q_heads * VF_D / 8;
      for (int k = threadIdx.x; k < n; k += VF_THREADS) o[k] = make_uint4(0, 0, 0, 0);
    }
  }
  if (ua >= ub) return;  // no unit for this CTA: leave before taking tensor memory
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh.tmem_base)),
                 "r"(VF_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0 || warp == 2) {
    // ================================================================ TMA producers
    // warp 0 loads Q (per item) and K tiles, warp 2 the V tiles: each ring
    // refills as soon as its own stage is free
    const bool is_k = warp == 0;
    const int nst = is_k ? L::KST : L::VST;
    uint64_t* full = is_k ? sh.k_full : sh.v_full;
    uint64_t* empty = is_k ? sh.k_empty : sh.v_empty;
    const CUtensorMap* tm = is_k ? &tmk : &tmv;
    uint8_t* ring = smem + (is_k ? L::K_OFF : L::V_OFF);
    if (lane == 0) {
      if (is_k) prefetch_tmap(&tmq);
      prefetch_tmap(tm);
    }
    const uint64_t pol = policy_evict_first();  // each K/V tile is read once
    // lane b < 8: block and row offset of keys 128 j + 16 b .. + 15 of item x
    auto tile_ids = [&](const VfItem& x, int j, int& blk, int& y) {
      blk = -1;
      y = 0;
      if (lane < VF_N / 16) {
        const int key0 = j * VF_N + lane * 16;
        const int lb = key0 / p.block_size;
        y = key0 - lb * p.block_size;
        if (lb < (x.ctx + p.block_size - 1) / p.block_size) {
          blk = __ldg(p.block_tables + static_cast<long long>(x.s) * p.max_blocks + lb);
          if (is_k && (blk < 0 || blk >= p.num_blocks)) set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
        }
      }
    };
    uint32_t g = 0, i = 0;  // tiles issued, items
    bool ok = true;
    VfItem it;
    vf_seek(p, pfx, ua, ua, ub, it);
    do {
      if (is_k) {
        const int qb = i & 1;
        if (i >= 2 && !(ok = vf_wait(sh, &sh.q_empty[qb], ((i >> 1) - 1) & 1, p.status))) break;
        if (lane == 0) {
          uint8_t* dq = smem + L::Q_OFF + qb * L::QBUF;
          mbar_arrive_expect_tx(&sh.q_full[qb], L::QBUF);
          tma_load_3d(dq, &tmq, &sh.q_full[qb], 0, it.kvh * p.group, it.q0);
          tma_load_3d(dq + L::QP, &tmq, &sh.q_full[qb], 64, it.kvh * p.group, it.q0);
        }
      }
      int blk, y;
      tile_ids(it, it.t0, blk, y);
      for (int j = it.t0; j < it.t1; ++j) {
        int nblk = -1, ny = 0;
        if (j + 1 < it.t1) tile_ids(it, j + 1, nblk, ny);  // the next tile's table entry loads during the wait
        const int st = g % nst;
        if (g >= static_cast<uint32_t>(nst) && !(ok = vf_wait(sh, &empty[st], ((g / nst) - 1) & 1, p.status))) break;
        if (lane == 0) mbar_arrive_expect_tx(&full[st], VF_KV_BYTES);
        __syncwarp();
        if (lane < VF_N / 16) {  // out-of-range block IDs read zeros (and were reported)
          uint8_t* dst = ring + st * VF_KV_BYTES + lane * 2048;
          tma_load_4d(dst, tm, &full[st], 0, y, it.kvh, blk, pol);
          tma_load_4d(dst + VF_PANEL, tm, &full[st], 64, y, it.kvh, blk, pol);
        }
        ++g;
        blk = nblk;
        y = ny;
      }
      if (!ok) break;
      ++i;
    } while (!sh.abort && vf_next(p, pfx, ua, ub, it));
    if (sh.abort) {  // let this warp's copies still in flight land before shared memory goes away
      for (int st = 0; st < nst; ++st) {
        const uint32_t uses = g / nst + (static_cast<uint32_t>(st) < g % nst ? 1u : 0u);
        if (uses > 0) mbar_wait(&full[st], (uses - 1) & 1);
      }
      if (is_k) {
        for (uint32_t b = 0; b < 2; ++b) {
          const uint32_t uses = i / 2 + (b < i % 2 ? 1u : 0u);
          if (uses > 0) mbar_wait(&sh.q_full[b], (uses - 1) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // Issues S(g) and P V(g) as their inputs become ready (non-blocking
    // tests), S running ahead of P V: the next tile's S is computed while the
    // softmax works on the current one.  The warp gives up after WAIT_NS
    // without progress.
    const uint32_t idesc_s = umma_idesc(VF_N, NCOL, 0, 0);  // S^T = K Q^T: M = keys, N = columns
    const uint32_t idesc_o = umma_idesc(128, VF_D, 0, 1);   // O = P V: M = columns (of 128), N = head_dim
    const uint32_t sbase = smem_u32(smem);
    constexpr int RING = 4;           // tiles whose S is issued and P V is not
    uint32_t job_item[RING];          // their item (its O slot and the o_empty phase)
    bool job_first[RING];             // their P V starts the item's O
    bool o_first = true;
    uint32_t gs = 0, is = 0, gp = 0;  // next S tile, its item; next P V tile
    VfItem it;
    vf_seek(p, pfx, ua, ua, ub, it);
    int j = it.t0;
    bool s_more = true;
    uint64_t t_idle = globaltimer_ns();
    uint32_t spins = 0;
    while (true) {
      bool prog = false;
      if (s_more && gs - gp < static_cast<uint32_t>(RING)) {
        const int ks = gs % L::KST, b = gs & 1, qb = is & 1;
        bool rdy = (j != it.t0 || mbar_test_wait(&sh.q_full[qb], (is >> 1) & 1)) &&
                   mbar_test_wait(&sh.k_full[ks], (gs / L::KST) & 1) &&
                   (gs < 2 || mbar_test_wait(&sh.s_empty[b], ((gs >> 1) - 1) & 1));
        rdy = __shfl_sync(FULL_MASK, rdy, 0);
        if (rdy) {
          tc_fence_after();
          const uint32_t sk = sbase + L::K_OFF + ks * VF_KV_BYTES;
          const uint32_t sq = sbase + L::Q_OFF + qb * L::QBUF;
#pragma unroll
          for (int kk = 0; kk < VF_D / 16; ++kk) {
            const uint32_t offk = (kk >> 2) * VF_PANEL + (kk & 3) * 32, offq = (kk >> 2) * L::QP + (kk & 3) * 32;
            umma_f16(tmem + b * NCOL, umma_desc(sk + offk, 16, 1024), umma_desc(sq + offq, 16, 1024), idesc_s,
                     kk > 0 ? 1u : 0u);
          }
          umma_commit(&sh.s_full[b]);
          umma_commit(&sh.k_empty[ks]);
          if (j == it.t1 - 1) umma_commit(&sh.q_empty[qb]);
          job_item[gs % RING] = is;
          job_first[gs % RING] = o_first;
          o_first = false;
          ++gs;
          prog = true;
          if (++j == it.t1) {
            ++is;
            if (vf_next(p, pfx, ua, ub, it)) {
              j = it.t0;
              o_first = true;
            } else {
              s_more = false;
            }
          }
        }
      }
      if (gp < gs) {
        const int b = gp & 1, vs = gp % L::VST;
        const uint32_t ji = job_item[gp % RING];
        const bool first = job_first[gp % RING];
        const int os = ji & 1;  // O slot: one per item parity
        bool rdy = mbar_test_wait(&sh.p_full[b], (gp >> 1) & 1) && mbar_test_wait(&sh.v_full[vs], (gp / L::VST) & 1);
        // the item two back, which used this O, has had its epilogue
        if (rdy && first && ji >= 2) rdy = mbar_test_wait(&sh.o_empty[os], ((ji >> 1) - 1) & 1);
        rdy = __shfl_sync(FULL_MASK, rdy, 0);
        if (rdy) {
          tc_fence_after();
          const uint32_t sp = sbase + L::P_OFF;
          const uint32_t sv = sbase + L::V_OFF + vs * VF_KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < VF_N / 16; ++kk)  // keys 16 kk .. + 15: P columns of panel kk / 4, V rows 16 kk ..
            umma_f16(tmem + VF_TMEM_O + os * 128, umma_desc(sp + (kk >> 2) * L::PP + (kk & 3) * 32, 16, 1024),
                     umma_desc(sv + kk * 16 * 128, VF_PANEL, 1024), idesc_o, (!first || kk > 0) ? 1u : 0u);
          umma_commit(&sh.pv_done[b]);
          umma_commit(&sh.v_empty[vs]);
          ++gp;
          prog = true;
        }
      }
      if (!s_more && gp == gs) break;
      if (prog) {
        spins = 0;
        t_idle = globaltimer_ns();
      } else if ((++spins & 63) == 0) {
        if (*reinterpret_cast<volatile int*>(&sh.abort)) break;
        if (globaltimer_ns() - t_idle > WAIT_NS) {
          sh.abort = 1;
          set_status(p.status, PA_STATUS_BIT(PA_ERR_TIMEOUT));
          break;
        }
      }
    }
  } else if (warp >= 4) {
    // ================================================================ softmax + epilogue
    // The four warps meet at a named barrier, which cannot time out: none of
    // them leaves the item loop early.  A failed wait only records itself (the
    // first one raises the abort flag, after which every wait returns at once)
    // and the loop runs on over the remaining items without merging pieces.
    const int quad = warp & 3;                // TMEM lane quadrant of this warp
    const int t = quad * 32 + lane;           // key of the tile = TMEM lane of S^T; column of O
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    float* red = reinterpret_cast<float*>(smem + L::RED_OFF);  // [2][4][NCOL]
    float* lred = red + 2 * 4 * NCOL;                          // [4][NCOL]
    float* mvs = lred + 4 * NCOL;                              // [4][NCOL]: -m (0 for a column with no key yet)
    float* avs = mvs + 4 * NCOL;                               // [4][NCOL]
    float* em = avs + 4 * NCOL;                                // [2][NCOL]
    float* el = em + 2 * NCOL;                                 // [2][NCOL]
    const float cs = p.scale_log2;
    const int G = p.group;
    uint32_t g = 0, i = 0;
    bool ok = true;

    // An item's epilogue runs once its last P V has completed: after the
    // softmax of the next tile has waited for that P V (so the item's end
    // never stalls the next item's tiles), or at the end of the range.
    VfItem pend;
    uint32_t pend_g = 0, pend_i = 0;
    bool pending = false;
    auto finish = [&](bool wait) {
      if (wait) ok = vf_wait(sh, &sh.pv_done[pend_g & 1], (pend_g >> 1) & 1, p.status) && ok;
      tc_fence_after();
      const int ps = pend_i & 1;
      const bool cut = pend.t0 > 0 || pend.t1 < pend.nt;
      const int ncolv = pend.qlen * G;
      const int b0 = vf_cta_of(pend.base, T, nct), b1 = vf_cta_of(pend.base + pend.nt - 1, T, nct);
      if (quad < NC32) {  // thread t owns column t of O
        const float mcol = em[ps * NCOL + t], lsum = el[ps * NCOL + t];
        const uint32_t o_addr = tmem + lane_base + VF_TMEM_O + ps * 128;
        if (!cut) {
          const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
          __nv_bfloat16* orow =
              static_cast<__nv_bfloat16*>(p.out) +
              (static_cast<long long>(pend.q0 + t / G) * p.num_q_heads + pend.kvh * G + t % G) * VF_D;
#pragma unroll
          for (int k = 0; k < VF_D / 32; ++k) {
            float v[32];
            tmem_ld32(o_addr + 32 * k, v);
            tmem_wait_ld();
            if (t < ncolv) {
#pragma unroll
              for (int c = 0; c < 32; c += 8) {
                uint4 u;
                u.x = pack_bf16x2(v[c] * inv, v[c + 1] * inv);
                u.y = pack_bf16x2(v[c + 2] * inv, v[c + 3] * inv);
                u.z = pack_bf16x2(v[c + 4] * inv, v[c + 5] * inv);
                u.w = pack_bf16x2(v[c + 6] * inv, v[c + 7] * inv);
                *reinterpret_cast<uint4*>(orow + 32 * k + c) = u;
              }
            }
          }
        } else {
          // this CTA's piece: its first item goes to slot 0, its last to slot 1
          const int slot = pend.base <= ua ? 0 : 1;
          float* ps_ = p.slots + (static_cast<long long>(blockIdx.x) * 2 + slot) * verify_slot_floats(NCOL);
#pragma unroll
          for (int k = 0; k < VF_D / 32; ++k) {
            float v[32];
            tmem_ld32(o_addr + 32 * k, v);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4*>(ps_ + t * VF_D + 32 * k + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
          }
          ps_[NCOL * VF_D + t] = mcol;
          ps_[NCOL * VF_D + NCOL + t] = lsum;
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.o_empty[ps]);
      if (cut) {
        // the CTA that lands the last piece of the item merges all of them, in CTA order
        __threadfence();
        softmax_bar();
        if (t == 0) {
          // pieces: the CTAs b0 .. b1 whose ranges are not empty (with fewer
          // units than CTAs some ranges are)
          int pieces = 0;
          for (int bb = b0; bb <= b1; ++bb) pieces += vf_range_start(bb + 1, T, nct) > vf_range_start(bb, T, nct);
          const int prev = atomicAdd(p.counters + b1, 1);
          sh.merge = prev == pieces - 1 && !*reinterpret_cast<volatile int*>(&sh.abort);
        }
        softmax_bar();
        if (sh.merge) {
          __threadfence();
          // thread t: column t % NCOL, head-dims [d0, d0 + DPER) of it; every
          // piece's values load as independent vectors
          constexpr int DPER = VF_D * NCOL / 128;
          const int c = t % NCOL, d0 = (t / NCOL) * DPER;
          const long long r0 = vf_range_start(b0, T, nct);
          auto piece = [&](int bb) -> const float* {
            const int sl = (bb == b0 && pend.base != r0) ? 1 : 0;
            return p.slots + (static_cast<long long>(bb) * 2 + sl) * verify_slot_floats(NCOL);
          };
          if (c < ncolv) {
            float mx = -INFINITY;
            for (int bb = b0; bb <= b1; ++bb) {
              if (vf_range_start(bb + 1, T, nct) == vf_range_start(bb, T, nct)) continue;  // empty range
              mx = fmaxf(mx, __ldcg(piece(bb) + NCOL * VF_D + c));
            }
            __nv_bfloat16* orow =
                static_cast<__nv_bfloat16*>(p.out) +
                (static_cast<long long>(pend.q0 + c / G) * p.num_q_heads + pend.kvh * G + c % G) * VF_D + d0;
#pragma unroll 1
            for (int dc = 0; dc < DPER; dc += 32) {
              float acc[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) acc[e] = 0.f;
              float lt = 0.f;
              for (int bb = b0; bb <= b1; ++bb) {
                if (vf_range_start(bb + 1, T, nct) == vf_range_start(bb, T, nct)) continue;
                const float* q = piece(bb);
                const float m = __ldcg(q + NCOL * VF_D + c);
                const float wgt = m == -INFINITY ? 0.f : fast_exp2(m - mx);
                lt += __ldcg(q + NCOL * VF_D + NCOL + c) * wgt;
                const float4* o4 = reinterpret_cast<const float4*>(q + c * VF_D + d0 + dc);
                float4 v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = __ldcg(o4 + e);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  acc[4 * e] += v[e].x * wgt;
                  acc[4 * e + 1] += v[e].y * wgt;
                  acc[4 * e + 2] += v[e].z * wgt;
                  acc[4 * e + 3] += v[e].w * wgt;
                }
              }
              const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll
              for (int e = 0; e < 32; e += 8) {
                uint4 u;
                u.x = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
                u.y = pack_bf16x2(acc[e + 2] * inv, acc[e + 3] * inv);
                u.z = pack_bf16x2(acc[e + 4] * inv, acc[e + 5] * inv);
                u.w = pack_bf16x2(acc[e + 6] * inv, acc[e + 7] * inv);
                *reinterpret_cast<uint4*>(orow + dc + e) = u;
              }
            }
          }
          if (t == 0) p.counters[b1] = 0;  // back to zero for the next call
        }
        softmax_bar();
        if (t == 0) sh.merge = 0;
      }
      pending = false;
    };

    VfItem it;
    vf_seek(p, pfx, ua, ua, ub, it);
    do {
      const uint32_t o_addr = tmem + lane_base + VF_TMEM_O + (i & 1) * 128;  // this item's O
      const int p0 = it.ctx - it.qlen;
      float mr[NC32];  // running reference maxima of columns lane + 32 k (the same in every warp)
      float lp[NCOL];  // this key lane's share of each column's sum
#pragma unroll
      for (int k = 0; k < NC32; ++k) mr[k] = -INFINITY;
#pragma unroll
      for (int c = 0; c < NCOL; ++c) lp[c] = 0.f;
      uint32_t g_last = 0;
      for (int j = it.t0; j < it.t1; ++j, ++g) {
        const int b = g & 1;
        const uint32_t s_addr = tmem + lane_base + b * NCOL;
        ok = vf_wait(sh, &sh.s_full[b], (g >> 1) & 1, p.status) && ok;
        tc_fence_after();
        // column c is visible to this key iff c >= cthr (rows i >= key - p0; keys past the context: none)
        const int key = j * VF_N + t, kr = key - p0;
        const int cthr = kr <= 0 ? 0 : (kr < it.qlen ? kr * G : NCOL);
        const bool diag = j * VF_N + VF_N - 1 - p0 > 0;
        // ---- column maxima: reduce-scatter in the warp, then across the four warps
        constexpr bool kReload = NCOL > 32;  // 64 columns: the registers go to the reduction, S is read again
        float x[NCOL];
        auto load_scaled = [&]() {
#pragma unroll
          for (int k = 0; k < NC32; ++k) {
            float v[32];
            tmem_ld32(s_addr + 32 * k, v);
#pragma unroll
            for (int c = 0; c < 32; ++c) x[32 * k + c] = v[c] * cs;
          }
          tmem_wait_ld();
          if (diag) {
#pragma unroll
            for (int c = 0; c < NCOL; ++c) x[c] = c < cthr ? -INFINITY : x[c];
          }
        };
        if constexpr (kReload) {
#pragma unroll
          for (int k = 0; k < NC32; ++k) {
            float v[32];
            tmem_ld32(s_addr + 32 * k, v);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] *= cs;
            if (diag) {
#pragma unroll
              for (int c = 0; c < 32; ++c) v[c] = 32 * k + c < cthr ? -INFINITY : v[c];
            }
            red[(b * 4 + quad) * NCOL + 32 * k + lane] = vf_reduce_scatter32<true>(v, lane);
          }
        } else {
          load_scaled();
          tc_fence_before();
          mbar_arrive(&sh.s_empty[b]);  // S_b may now take tile g + 2
          float v[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = x[c];
          red[(b * 4 + quad) * NCOL + lane] = vf_reduce_scatter32<true>(v, lane);
        }
        softmax_bar();
        bool moved = false;
#pragma unroll
        for (int k = 0; k < NC32; ++k) {
          const int c = 32 * k + lane;
          const float tm = fmaxf(fmaxf(red[(b * 4 + 0) * NCOL + c], red[(b * 4 + 1) * NCOL + c]),
                                 fmaxf(red[(b * 4 + 2) * NCOL + c], red[(b * 4 + 3) * NCOL + c]));
          const float mo = mr[k];
          const float mn = (tm > mo + VF_RESCALE_LOG2 || mo == -INFINITY) ? fmaxf(tm, mo) : mo;
          avs[quad * NCOL + c] = (mo == -INFINITY || mn == mo) ? 1.f : fast_exp2(mo - mn);
          moved |= mn != mo;
          mr[k] = mn;
          mvs[quad * NCOL + c] = mn == -INFINITY ? 0.f : -mn;  // a column with no key yet: P = 0
        }
        const bool resc = __any_sync(FULL_MASK, moved);  // the same in every warp
        __syncwarp();
        if constexpr (kReload) {
          load_scaled();
          tc_fence_before();
          mbar_arrive(&sh.s_empty[b]);
        }
        const bool had = j > it.t0;  // O already holds earlier tiles of this item
        if (resc) {
#pragma unroll
          for (int c = 0; c < NCOL; c += 4) {
            const float4 a = *reinterpret_cast<const float4*>(avs + quad * NCOL + c);
            lp[c] *= a.x;
            lp[c + 1] *= a.y;
            lp[c + 2] *= a.z;
            lp[c + 3] *= a.w;
          }
        }
        // P = exp2(S - m) by 32 columns; P last fed P V(g - 1): wait for it
        // (after the first 32 exponentials) before overwriting
        {
          uint8_t* pb = smem + L::P_OFF + (t >> 6) * L::PP;
          const int kc = (t & 63) >> 3, ke = (t & 7) * 2;
#pragma unroll
          for (int k = 0; k < NC32; ++k) {
            float pr[32];
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              const float4 nm = *reinterpret_cast<const float4*>(mvs + quad * NCOL + 32 * k + c);
              pr[c] = fast_exp2(x[32 * k + c] + nm.x);
              pr[c + 1] = fast_exp2(x[32 * k + c + 1] + nm.y);
              pr[c + 2] = fast_exp2(x[32 * k + c + 2] + nm.z);
              pr[c + 3] = fast_exp2(x[32 * k + c + 3] + nm.w);
#pragma unroll
              for (int e = 0; e < 4; ++e) lp[32 * k + c + e] += pr[c + e];
            }
            if (k == 0 && g >= 1) ok = vf_wait(sh, &sh.pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, p.status) && ok;
#pragma unroll
            for (int c = 0; c < 32; ++c)
              *reinterpret_cast<__nv_bfloat16*>(pb + (32 * k + c) * 128 + ((kc ^ (c & 7)) << 4) + ke) =
                  __float2bfloat16_rn(pr[c]);
          }
        }
        // keys past the context may hold anything (even NaN): zero their V rows
        const int valid = it.ctx - j * VF_N;
        if (valid < VF_N) {
          const int vs = g % L::VST;
          ok = vf_wait(sh, &sh.v_full[vs], (g / L::VST) & 1, p.status) && ok;
          if (t >= valid) {  // chunks in a lane-rotated order: the 32 lanes spread over the banks
            uint8_t* vrow = smem + L::V_OFF + vs * VF_KV_BYTES + t * 128;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int ch = (k + t) & 7;
              *reinterpret_cast<uint4*>(vrow + ch * 16) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(vrow + VF_PANEL + ch * 16) = make_uint4(0, 0, 0, 0);
            }
          }
        }
        if (resc && had) {
          // O holds this item's earlier tiles: wait for the last P V into it
          // (tile g - 1), then scale row t of O (column t) before P V(g) adds to it
          ok = vf_wait(sh, &sh.pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, p.status) && ok;
          tc_fence_after();
          if (quad < NC32) {
            const float a = avs[quad * NCOL + t];
#pragma unroll
            for (int k = 0; k < VF_D / 32; ++k) {
              float v[32];
              tmem_ld32(o_addr + 32 * k, v);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) v[c] *= a;
              tmem_st32(o_addr + 32 * k, v);
            }
            tmem_wait_st();
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sh.p_full[b]);
        g_last = g;
        // the P wait above covered P V(g - 1): the epilogue of an item that
        // ended there can run now without waiting
        if (pending && g == pend_g + 1) finish(false);
      }

      // ---- end of the item: column sums now, the rest of the epilogue deferred
#pragma unroll
      for (int k = 0; k < NC32; ++k) {
        float v[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = lp[32 * k + c];
        lred[quad * NCOL + 32 * k + lane] = vf_reduce_scatter32<false>(v, lane);
      }
      softmax_bar();
      if (t < NCOL) {
        em[(i & 1) * NCOL + t] = (NC32 == 1 || quad == 0) ? mr[0] : mr[NC32 - 1];  // column t = lane + 32 quad
        el[(i & 1) * NCOL + t] = (lred[t] + lred[NCOL + t]) + (lred[2 * NCOL + t] + lred[3 * NCOL + t]);
      }
      pend = it;
      pend_g = g_last;
      pend_i = i;
      pending = true;
      ++i;
    } while (vf_next(p, pfx, ua, ub, it));  // every softmax warp walks every item: the named barriers stay matched
    if (pending) finish(true);
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(VF_TMEM_COLS) : "memory");
  }
}

// ------------------------------------------------------------------ host side

int verify_supported(int group, int head_dim, int num_seqs) {
  return head_dim == VF_D && num_seqs <= VERIFY_SMEM_SEQS &&
         (group == 1 || group == 2 || group == 4 || group == 8 || group == 16);
}

// q [Tq, Hq, D] bf16 as a 3-D tensor (D, Hq, Tq); box = 64 columns x G heads x NCOL/G tokens.
static int encode_vq_tmap(CUtensorMap* map, const void* q, int total_q_tokens, int num_q_heads, int group, int ncol,
                          EncodeTiledFn fn) {
  const cuuint64_t dims[3] = {VF_D, static_cast<cuuint64_t>(num_q_heads), static_cast<cuuint64_t>(total_q_tokens)};
  const cuuint64_t strides[2] = {VF_D * 2, static_cast<cuuint64_t>(num_q_heads) * VF_D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(ncol / group)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : cu_fail(r, "cuTensorMapEncodeTiled");
}

template <int NCOL>
static int launch_verify_t(const VerifyParams& p0, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv, cudaStream_t stream, int num_sms) {
  auto kern = verify_kernel<NCOL>;
  const int smem = VfLayout<NCOL>::BYTES + 1024;
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
  VerifyParams p = p0;
  p.ncol_lo = NCOL == 32 ? 0 : 32;
  p.ncol_hi = NCOL;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms));  // one CTA per SM, one contiguous unit range each
  cfg.blockDim = dim3(VF_THREADS);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return check_launch(cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p), "verify_kernel launch");
}

int launch_verify(const VerifyParams& p, const void* q, const void* k_cache, const void* v_cache,
                  int total_q_tokens, cudaStream_t stream, int num_sms, int which) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return PA_ERR_CUDA;
  CUtensorMap tk, tv;
  int rc;
  if ((rc = encode_kv16_tmap(&tk, k_cache, p.num_blocks, p.num_kv_heads, p.block_size, VF_D, fn)) != PA_OK) return rc;
  if ((rc = encode_kv16_tmap(&tv, v_cache, p.num_blocks, p.num_kv_heads, p.block_size, VF_D, fn)) != PA_OK) return rc;
  // columns <= 32 on the 32-wide kernel, 33 .. 64 on the 64-wide one
  CUtensorMap tq;
  if (which & 1) {
    if ((rc = encode_vq_tmap(&tq, q, total_q_tokens, p.num_q_heads, p.group, 32, fn)) != PA_OK) return rc;
    if ((rc = launch_verify_t<32>(p, tq, tk, tv, stream, num_sms)) != PA_OK) return rc;
  }
  if (which & 2) {
    if ((rc = encode_vq_tmap(&tq, q, total_q_tokens, p.num_q_heads, p.group, 64, fn)) != PA_OK) return rc;
    if ((rc = launch_verify_t<64>(p, tq, tk, tv, stream, num_sms)) != PA_OK) return rc;
  }
  return PA_OK;
}

}  // namespace pa
