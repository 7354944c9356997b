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
//  * M-tile = 128 query rows = 128/G consecutive tokens x the G query heads of
//    one KV head (GQA packing: every K/V tile feeds all G heads).  Q comes in
//    with one 3-D TMA box per head-dim half (128 rows x 128 bytes, 128-byte
//    swizzle) -- a K-major UMMA operand as it lands.
//  * N-tile = 128 keys: 128/block_size blocks, each fetched with 16-row TMA
//    boxes straight into K-major SW128 panels (K for S = Q K^T) and the same
//    panels serve as the MN-major B operand of O += P V.
//  * Warp roles (6 warps): warp 0 issues TMA; warp 1 allocates tensor memory
//    and issues tcgen05.mma from one thread; warps 2-5 (128 threads, thread =
//    TMEM lane = query row) run the softmax.  S is double-buffered in TMEM so
//    QK^T of tile j+1 overlaps the softmax of tile j; O (128 fp32 columns)
//    stays in TMEM for the whole M-tile.
//  * Softmax: row max and exp2 on the thread's own row (no shuffles), causal
//    mask on diagonal tiles only, O is rescaled in TMEM only when the running
//    maximum rises by more than 2^8 (between rescales the stale maximum is an
//    exact reference point).  P goes to shared memory as a K-major SW128 A
//    operand.  Key rows past the context are zeroed in V before P V.
//  * Every wait is bounded; on a timeout the CTA raises PA_ERR_TIMEOUT, stops
//    all roles through a shared abort flag, drains its tensor-core work and
//    frees its tensor memory.
#include <cuda.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int CH_THREADS = 192;
constexpr int CH_D = 128;
constexpr int CH_M = 128;                   // query rows per M-tile
constexpr int CH_N = 128;                   // keys per N-tile
constexpr int PANEL = CH_M * 128;           // one 128-row x 128-byte swizzled panel (16 KB)
constexpr int Q_BYTES = 2 * PANEL;          // [2 head-dim halves][128 rows][128 B]
constexpr int KV_BYTES = 2 * PANEL;         // one K (or V) tile
constexpr int KST = 3;                      // K stages (a K tile is free once its QK^T is done)
constexpr int VST = 2;                      // V stages (a V tile is free once its PV is done)
constexpr int SMEM_Q = 0;
constexpr int SMEM_K = SMEM_Q + Q_BYTES;
constexpr int SMEM_V = SMEM_K + KST * KV_BYTES;
constexpr int SMEM_P = SMEM_V + VST * KV_BYTES;
constexpr int SMEM_TOTAL = SMEM_P + Q_BYTES;                  // + P (same shape as Q): 224 KB
constexpr uint32_t TMEM_COLS = 512;                           // S0 [0,128), S1 [128,256), O [256,384)
constexpr uint32_t TMEM_O = 256;
constexpr float RESCALE_LOG2 = 8.f;                           // rescale O when the max rises by > 2^8

// ---- tcgen05 / UMMA helpers
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  // shared-memory matrix descriptor: start >> 4, LBO >> 4, SBO >> 4, version 1, 128-byte swizzle
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFF) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16 instruction descriptor: bf16 x bf16 -> fp32, M x N, A/B major-ness
__device__ __forceinline__ constexpr uint32_t umma_idesc(int m, int n, int a_mn_major, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn_major) << 15) |
         (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])),
      "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
      "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
      "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
      "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
      "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

struct Item {
  int s;           // sequence
  int q0, qlen;    // its query rows
  int p0, ctx;     // position of its first row, its key count
  int tb, kvh;     // token block (of 128/G tokens) and KV head
};

struct Shared {
  uint64_t q_full, q_empty, o_empty, pv_done, drain;
  uint64_t s_full[2], s_empty[2];
  uint64_t k_full[KST], k_empty[KST], v_full[VST], v_empty[VST];
  uint64_t p_full;
  uint32_t tmem_base;
  int abort;
  long long total;
};

}  // namespace

// Items = (multi-row sequence, token block, KV head), numbered sequence by
// sequence; every CTA walks items blockIdx.x, + gridDim.x, ...  The batch is
// scanned from global memory by each role (it is small and L1-resident).
__device__ __forceinline__ bool chunk_item(const ChunkParams& p, int tok, long long idx, Item& it) {
  long long base = 0;
  for (int s = 0; s < p.num_seqs; ++s) {
    const int q0 = __ldg(p.query_start + s), qlen = __ldg(p.query_start + s + 1) - q0;
    if (qlen <= 1) continue;
    int ctx = __ldg(p.context_lens + s);
    const int cap = p.max_blocks * p.block_size;
    if (ctx > cap) ctx = cap;
    const int nblk = (qlen + tok - 1) / tok;
    const long long n = static_cast<long long>(nblk) * p.num_kv_heads;
    if (idx < base + n) {
      const int r = static_cast<int>(idx - base);
      it.s = s;
      it.q0 = q0;
      it.qlen = qlen;
      it.ctx = ctx;
      it.p0 = ctx - qlen;
      it.tb = r / p.num_kv_heads;
      it.kvh = r % p.num_kv_heads;
      return true;
    }
    base += n;
  }
  return false;
}

__device__ __forceinline__ long long chunk_total(const ChunkParams& p, int tok) {
  long long n = 0;
  for (int s = 0; s < p.num_seqs; ++s) {
    const int qlen = __ldg(p.query_start + s + 1) - __ldg(p.query_start + s);
    if (qlen > 1) n += static_cast<long long>((qlen + tok - 1) / tok) * p.num_kv_heads;
  }
  return n;
}

// Keys an item needs: up to the last position of its token block (capped at the context).
__device__ __forceinline__ int item_tiles(const Item& it, int tok) {
  int last = it.p0 + min((it.tb + 1) * tok, it.qlen) - 1;  // last visible key of the block's last row
  if (last >= it.ctx) last = it.ctx - 1;
  return last < 0 ? 0 : last / CH_N + 1;
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

template <int G>
__global__ void __launch_bounds__(CH_THREADS, 1)
    chunk_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                 const __grid_constant__ CUtensorMap tmv, const ChunkParams p) {
  constexpr int TOK = CH_M / G;  // tokens per M-tile
  extern __shared__ uint8_t smem_raw[];
  __shared__ Shared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sh.q_full, 1);
    mbar_init(&sh.q_empty, 1);
    mbar_init(&sh.o_empty, 128);
    mbar_init(&sh.pv_done, 1);
    mbar_init(&sh.drain, 1);
    mbar_init(&sh.p_full, 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.s_full[b], 1);
      mbar_init(&sh.s_empty[b], 128);
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
    sh.total = chunk_total(p, TOK);
    fence_mbar_init();
  }
  if (warp == 1) {  // tensor memory: S0, S1, O
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh.tmem_base)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  grid_dependency_wait();  // the cache may still be being appended by the kernel before this one

  const long long total = sh.total;
  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmq);
      prefetch_tmap(&tmk);
      prefetch_tmap(&tmv);
    }
    const uint64_t pol = policy_evict_last();  // a chunk's K/V is re-read by every M-tile of the chunk
    uint32_t items = 0, tcount = 0;  // tiles issued over all items (stage and phase bookkeeping)
    for (long long idx = blockIdx.x; idx < total && !sh.abort; idx += gridDim.x, ++items) {
      Item it;
      if (!chunk_item(p, TOK, idx, it)) break;
      const int nt = item_tiles(it, TOK);
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
      tile_ids(0, blk_cur, y_cur);
      tile_ids(1, blk_next, y_next);
      // the previous item's last QK^T has read Q
      if (items > 0 && !ch_wait(sh, &sh.q_empty, (items - 1) & 1, p.status)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&sh.q_full, Q_BYTES);
        tma_load_3d(smem + SMEM_Q, &tmq, &sh.q_full, 0, it.kvh * G, it.q0 + it.tb * TOK);
        tma_load_3d(smem + SMEM_Q + PANEL, &tmq, &sh.q_full, 64, it.kvh * G, it.q0 + it.tb * TOK);
      }
      auto load_tile = [&](const CUtensorMap* tm, uint64_t* bars_full, uint64_t* bars_empty, int nst, int base_off,
                           uint32_t t, int blk, int y) -> bool {
        const int st = t % nst;
        const uint32_t use = t / nst;  // earlier fills of this stage
        if (use > 0 && !ch_wait(sh, &bars_empty[st], (use - 1) & 1, p.status)) return false;
        if (lane == 0) mbar_arrive_expect_tx(&bars_full[st], KV_BYTES);
        __syncwarp();
        if (lane < CH_N / 16) {  // 16-row boxes (head-dim half, 16 keys) -> rows 16*lane.. of both panels
          if (blk >= p.num_blocks) set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
          uint8_t* dst = smem + base_off + st * KV_BYTES + lane * 2048;
          tma_load_4d(dst, tm, &bars_full[st], 0, y, it.kvh, blk, pol);
          tma_load_4d(dst + PANEL, tm, &bars_full[st], 64, y, it.kvh, blk, pol);
        }
        return true;
      };
      bool ok = true;
      for (int j = 0; ok && j < nt; ++j) {
        ok = load_tile(&tmk, sh.k_full, sh.k_empty, KST, SMEM_K, tcount + j, blk_cur, y_cur);
        if (ok && j > 0) ok = load_tile(&tmv, sh.v_full, sh.v_empty, VST, SMEM_V, tcount + j - 1, blk_prev, y_prev);
        blk_prev = blk_cur;
        y_prev = y_cur;
        blk_cur = blk_next;
        y_cur = y_next;
        tile_ids(j + 2, blk_next, y_next);  // one tile of lead for the block-table reads
      }
      if (ok && nt > 0) ok = load_tile(&tmv, sh.v_full, sh.v_empty, VST, SMEM_V, tcount + nt - 1, blk_prev, y_prev);
      tcount += nt;
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
    const uint32_t idesc_pv = umma_idesc(CH_M, CH_D, 0, 1);
    const uint32_t sq = smem_u32(smem + SMEM_Q), sp = smem_u32(smem + SMEM_P);
    uint32_t q_phase = 0, p_phase = 0, o_phase = 0, s_use[2] = {0, 0}, kv_count = 0;
    bool first_item = true;
    for (long long idx = blockIdx.x; idx < total && !sh.abort; idx += gridDim.x) {
      Item it;
      if (!chunk_item(p, TOK, idx, it)) break;
      const int nt = item_tiles(it, TOK);
      if (!ch_wait(sh, &sh.q_full, q_phase, p.status)) break;
      q_phase ^= 1;
      if (!first_item) {  // the epilogue of the previous item has read O
        if (!ch_wait(sh, &sh.o_empty, o_phase, p.status)) break;
        o_phase ^= 1;
      }
      first_item = false;
      bool ok = true;
      auto qk = [&](int j) -> bool {
        const int stage = (kv_count + j) % KST;
        const uint32_t use = (kv_count + j) / KST;
        if (!ch_wait(sh, &sh.k_full[stage], use & 1, p.status)) return false;
        const int sb = j & 1;
        if (s_use[sb] > 0 && !ch_wait(sh, &sh.s_empty[sb], (s_use[sb] - 1) & 1, p.status)) return false;
        ++s_use[sb];
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sk = smem_u32(smem + SMEM_K + stage * KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < CH_D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * PANEL + (kk & 3) * 32;
            umma_f16(tmem + sb * CH_N, umma_desc(sq + off, 16, 1024), umma_desc(sk + off, 16, 1024), idesc_qk,
                     kk > 0);
          }
          umma_commit(&sh.s_full[sb]);
          umma_commit(&sh.k_empty[stage]);
          if (j == nt - 1) umma_commit(&sh.q_empty);
        }
        __syncwarp();
        return true;
      };
      auto pv = [&](int j) -> bool {
        if (!ch_wait(sh, &sh.p_full, p_phase, p.status)) return false;
        p_phase ^= 1;
        const int stage = (kv_count + j) % VST;
        if (!ch_wait(sh, &sh.v_full[stage], ((kv_count + j) / VST) & 1, p.status)) return false;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sv = smem_u32(smem + SMEM_V + stage * KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < CH_N / 16; ++kk) {
            // A = P (K-major, keys 16kk..), B = V (MN-major: 16 key rows from row 16kk, both head-dim panels)
            umma_f16(tmem + TMEM_O, umma_desc(sp + (kk >> 2) * PANEL + (kk & 3) * 32, 16, 1024),
                     umma_desc(sv + kk * 16 * 128, PANEL, 1024), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&sh.pv_done);
          umma_commit(&sh.v_empty[stage]);
        }
        __syncwarp();
        return true;
      };
      if (nt > 0) ok = qk(0);
      for (int j = 1; ok && j < nt; ++j) ok = qk(j) && pv(j - 1);
      if (ok && nt > 0) ok = pv(nt - 1);
      kv_count += nt;
      if (!ok) break;
    }
  } else {
    // ================================================================ softmax warpgroup
    const int quad = warp & 3;            // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;     // query row of the M-tile = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const int tok_in_tile = row / G, head_in_group = row % G;
    uint32_t s_phase[2] = {0, 0}, pv_phase = 0, kv_count = 0;
    uint8_t* pbuf = smem + SMEM_P;
    for (long long idx = blockIdx.x; idx < total && !sh.abort; idx += gridDim.x) {
      Item it;
      if (!chunk_item(p, TOK, idx, it)) break;
      const int nt = item_tiles(it, TOK);
      const int tok = it.tb * TOK + tok_in_tile;       // row's token within the chunk
      const int last_key = it.p0 + tok;                // causal limit (inclusive)
      const bool row_valid = tok < it.qlen && last_key >= 0;
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nt && ok; ++j) {
        const int sb = j & 1;
        if (!(ok = ch_wait(sh, &sh.s_full[sb], s_phase[sb], p.status))) break;
        s_phase[sb] ^= 1;
        tc_fence_after();
        float s[CH_N];
#pragma unroll
        for (int c = 0; c < CH_N / 32; ++c) {
          float v[32];
          tmem_ld32(tmem + lane_addr + sb * CH_N + c * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = v[i];
        }
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&sh.s_empty[sb]);

        const int key0 = j * CH_N;
        const bool diag = key0 + CH_N - 1 > it.p0 + it.tb * TOK;  // some row of the tile stops inside it
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
#pragma unroll
          for (int i = 8; i < CH_N; i += 8)
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = fmaxf(m8[k], s[i + k]);
          mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
          if (!diag) mx *= cs;
        }
        // Decide the reference maximum, compute P in registers (this overlaps the
        // previous tile's P V on the tensor cores), and only then wait for that
        // P V before P's shared memory is rewritten or O is rescaled.
        const bool rescale = mx > m_ref + RESCALE_LOG2 || m_ref == -INFINITY;
        const float m_new = rescale ? fmaxf(mx, m_ref) : m_ref;
        uint32_t pk[CH_N / 2];
        float l8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const float neg_m = -m_new;
#pragma unroll
        for (int i = 0; i < CH_N / 2; ++i) {
          const float x0 = s[2 * i], x1 = s[2 * i + 1];
          const float a = fast_exp2(diag ? x0 + neg_m : fmaf(x0, cs, neg_m));
          const float b = fast_exp2(diag ? x1 + neg_m : fmaf(x1, cs, neg_m));
          l8[i & 7] += a + b;
          pk[i] = pack_bf16x2(a, b);
        }
        if (j > 0) {
          if (!(ok = ch_wait(sh, &sh.pv_done, pv_phase, p.status))) break;
          pv_phase ^= 1;
          tc_fence_after();
        }
        if (rescale && m_ref != -INFINITY) {
          const float alpha = fast_exp2(m_ref - m_new);
          l *= alpha;
          if (j > 0) {  // O holds tiles 0..j-1: scale it in tensor memory
#pragma unroll
            for (int c = 0; c < CH_D / 32; ++c) {
              float v[32];
              tmem_ld32(tmem + lane_addr + TMEM_O + c * 32, v);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= alpha;
              tmem_st32(tmem + lane_addr + TMEM_O + c * 32, v);
            }
            tmem_wait_st();
          }
        }
        m_ref = m_new;
        l += ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
        // P (bf16), row `row` of the K-major SW128 A panels
#pragma unroll
        for (int c8 = 0; c8 < CH_N / 8; ++c8) {
          uint8_t* dst = pbuf + (c8 >> 3) * PANEL + sw128(row, c8 & 7);
          *reinterpret_cast<uint4*>(dst) = make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
        }
        // keys past the context may hold anything (even NaN): zero their V rows
        const int valid_keys = it.ctx - key0;
        if (valid_keys < CH_N) {
          const int stage = (kv_count + j) % VST;
          if (!(ok = ch_wait(sh, &sh.v_full[stage], ((kv_count + j) / VST) & 1, p.status))) break;
          uint8_t* vst = smem + SMEM_V + stage * KV_BYTES;
          const int nz = (CH_N - max(valid_keys, 0)) * 2 * 8;  // 16-byte chunks in both panels
          for (int k = threadIdx.x - 64; k < nz; k += 128) {
            const int r = max(valid_keys, 0) + k / 16, rest = k % 16;
            *reinterpret_cast<uint4*>(vst + (rest >> 3) * PANEL + r * 128 + (rest & 7) * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sh.p_full);
      }
      kv_count += nt;
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 -> out
      if (nt > 0) {
        if (!ch_wait(sh, &sh.pv_done, pv_phase, p.status)) break;
        pv_phase ^= 1;
        tc_fence_after();
      }
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) +
                            (static_cast<long long>(it.q0 + tok) * p.num_q_heads + it.kvh * G + head_in_group) * CH_D;
#pragma unroll
      for (int c = 0; c < CH_D / 32; ++c) {
        float v[32];
        if (nt > 0) {
          tmem_ld32(tmem + lane_addr + TMEM_O + c * 32, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        if (row_valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 w;
            w.x = pack_bf16x2(v[i] * inv, v[i + 1] * inv);
            w.y = pack_bf16x2(v[i + 2] * inv, v[i + 3] * inv);
            w.z = pack_bf16x2(v[i + 4] * inv, v[i + 5] * inv);
            w.w = pack_bf16x2(v[i + 6] * inv, v[i + 7] * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + i) = w;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.o_empty);
    }
  }

  // ---- teardown: drain this CTA's tensor-core work, then free tensor memory
  if (warp == 1) {
    if (lane == 0) umma_commit(&sh.drain);  // arrives once every MMA issued by this thread has completed
    __syncwarp();
    mbar_wait(&sh.drain, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

// ------------------------------------------------------------------ host side

int chunk_supported(int group, int head_dim) {
  return head_dim == CH_D && (group == 1 || group == 2 || group == 4 || group == 8 || group == 16);
}

// q [Tq, Hq, D] bf16 as a 3-D tensor (D, Hq, Tq); box = 64 columns x G heads x 128/G tokens.
static int encode_q_tmap(CUtensorMap* map, const void* q, int total_q_tokens, int num_q_heads, int group,
                         EncodeTiledFn fn) {
  const cuuint64_t dims[3] = {CH_D, static_cast<cuuint64_t>(num_q_heads), static_cast<cuuint64_t>(total_q_tokens)};
  const cuuint64_t strides[2] = {CH_D * 2, static_cast<cuuint64_t>(num_q_heads) * CH_D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(CH_M / group)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

// [num_blocks, Hkv, block_size, D] as a 4-D tensor; box = 64 columns x 16 rows of one (block, head).
static int encode_kv16_tmap(CUtensorMap* map, const void* cache, int num_blocks, int num_kv_heads, int block_size,
                            EncodeTiledFn fn) {
  const cuuint64_t row = CH_D * 2;
  const cuuint64_t dims[4] = {CH_D, static_cast<cuuint64_t>(block_size), static_cast<cuuint64_t>(num_kv_heads),
                              static_cast<cuuint64_t>(num_blocks)};
  const cuuint64_t strides[3] = {row, row * block_size, row * block_size * num_kv_heads};
  const cuuint32_t box[4] = {64, 16, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(cache), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

template <int G>
static int launch_chunk_t(const ChunkParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          cudaStream_t stream, int num_sms) {
  auto kern = chunk_kernel<G>;
  const int smem = SMEM_TOTAL + 1024;
  static int configured_dev = -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (configured_dev != dev) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return PA_ERR_CUDA;
    configured_dev = dev;
  }
  const int grid = num_sms;  // persistent: CTAs walk the items (their count is known on the device only)
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
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p) != cudaSuccess) return PA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int launch_chunk(const ChunkParams& p, const void* q, const void* k_cache, const void* v_cache, int total_q_tokens,
                 cudaStream_t stream, int num_sms) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return PA_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  int rc;
  if ((rc = encode_q_tmap(&tq, q, total_q_tokens, p.num_q_heads, p.group, fn)) != PA_OK) return rc;
  if ((rc = encode_kv16_tmap(&tk, k_cache, p.num_blocks, p.num_kv_heads, p.block_size, fn)) != PA_OK) return rc;
  if ((rc = encode_kv16_tmap(&tv, v_cache, p.num_blocks, p.num_kv_heads, p.block_size, fn)) != PA_OK) return rc;
  switch (p.group) {
    case 1: return launch_chunk_t<1>(p, tq, tk, tv, stream, num_sms);
    case 2: return launch_chunk_t<2>(p, tq, tk, tv, stream, num_sms);
    case 4: return launch_chunk_t<4>(p, tq, tk, tv, stream, num_sms);
    case 8: return launch_chunk_t<8>(p, tq, tk, tv, stream, num_sms);
    case 16: return launch_chunk_t<16>(p, tq, tk, tv, stream, num_sms);
    default: return PA_ERR_UNSUPPORTED;
  }
}

}  // namespace pa
