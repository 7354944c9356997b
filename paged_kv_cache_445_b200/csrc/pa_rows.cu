// pa_rows.cu -- attention of single query rows over the paged KV cache (the decode path).
//
// What it computes ("Inference optimization", AI Engineering from Scratch,
// Phase 10 / 12, sections "KV cache" and "Build it -- Step 2: attention with
// the KV cache"; "vLLM serving internals", Phase 17 / 04, "PagedAttention as a
// virtual memory system"): for query row r of sequence s at position p and
// query head h,  out = softmax_j(scale * q . K_j) V_j  over keys j = 0..p, the
// K/V rows gathered through the sequence's block table.  A decode row has
// p = context_len - 1.
//
// How (B200):
//  * Work unit = one 16-key tile of one (query row, KV head) "segment".  All
//    G = Hq / Hkv query heads of the KV head ride along, so each K/V byte is
//    read from HBM once per step.  Every warp scans context_lens itself,
//    computes the batch's total tile count T and takes an equal contiguous
//    range of it: the load balance is exact to one tile whatever the length
//    mix, and no host-side plan is needed.
//  * A segment cut by a range boundary is finished as partial (m, l, O)
//    results; the last warp to arrive (atomic counter in the workspace)
//    merges them, so there is no second launch and at most two partial
//    slots per warp.
//  * Tiles stream HBM -> shared memory through TMA (4-D tensor map over
//    [num_blocks, Hkv, block_size, D], block ID as a coordinate, 128-byte
//    swizzle), a ring of R stages per warp completed on mbarriers.  Each warp
//    is its own producer and consumer: no block-wide barriers.
//  * Math on the tensor cores with the legacy warp MMA (m16n8k16, bf16 in,
//    fp32 accumulate), keys in M and heads in N:  S^T[16 keys, 8 heads] =
//    K_tile . Q^T;  the online softmax runs on the S^T fragment;  P goes from
//    the accumulator layout to the B-operand layout with movmatrix; and
//    O^T[D, 8 heads] += V^T . P^T with V read by ldmatrix.trans.  G <= 8 uses
//    one 8-wide head tile, G <= 16 two.
#include <cuda.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

constexpr int TILE_KEYS = 16;
constexpr int ROWS_WARPS = 4;
constexpr int ROWS_THREADS = ROWS_WARPS * 32;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

__device__ __forceinline__ int ceil16(int n) { return (n + TILE_KEYS - 1) / TILE_KEYS; }

// sum_{k=1}^{n} ceil(k / 16): tiles of the rows whose key counts are 1..n.
__device__ __forceinline__ long long tiles_upto(int n) {
  if (n <= 0) return 0;
  const long long q = n >> 4, r = n & 15;
  return 8 * q * (q + 1) + r * (q + 1);
}

__device__ __forceinline__ long long warp_sum64(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL_MASK, v, o);
  return v;
}

__device__ __forceinline__ long long warp_incl_scan64(long long v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long n = __shfl_up_sync(FULL_MASK, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

struct SeqInfo {
  int ctx, qlen, q0;
};

__device__ __forceinline__ SeqInfo seq_info(const RowsParams& p, int s) {
  SeqInfo si;
  int ctx = __ldg(p.context_lens + s);
  if (p.query_start) {
    si.q0 = __ldg(p.query_start + s);
    si.qlen = __ldg(p.query_start + s + 1) - si.q0;
  } else {
    si.q0 = s;
    si.qlen = 1;
  }
  const int cap = p.max_blocks * p.block_size;
  if (ctx > cap) {
    set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
    ctx = cap;
  }
  si.ctx = ctx < 0 ? 0 : ctx;
  if (si.qlen < 0) si.qlen = 0;
  return si;
}

// Tiles of all (row, KV head) segments of one sequence.
__device__ __forceinline__ long long seq_units(const RowsParams& p, const SeqInfo& si) {
  if (p.skip_multi && si.qlen > 1) return 0;
  const int p0 = si.ctx - si.qlen;
  return static_cast<long long>(p.num_kv_heads) * (tiles_upto(si.ctx) - tiles_upto(p0 < 0 ? 0 : p0));
}

struct Cursor {
  int s, i, h, t;  // sequence, row within it, KV head, tile within the segment
  int n, nkeys;    // tiles and keys of the current segment
  int p0, qlen, q0;
  long long u;     // global unit index
};

__device__ __forceinline__ bool enter_seq(const RowsParams& p, Cursor& c, int s) {
  const SeqInfo si = seq_info(p, s);
  if (seq_units(p, si) == 0) return false;
  c.s = s;
  c.qlen = si.qlen;
  c.q0 = si.q0;
  c.p0 = si.ctx - si.qlen;
  c.i = c.p0 < 0 ? -c.p0 : 0;  // first row that has a key
  c.h = 0;
  c.t = 0;
  c.nkeys = c.p0 + c.i + 1;
  c.n = ceil16(c.nkeys);
  return true;
}

__device__ __forceinline__ void advance(const RowsParams& p, Cursor& c) {
  ++c.u;
  if (++c.t < c.n) return;
  c.t = 0;
  if (++c.h < p.num_kv_heads) return;
  c.h = 0;
  if (++c.i < c.qlen) {
    ++c.nkeys;
    c.n = ceil16(c.nkeys);
    return;
  }
  for (int s = c.s + 1; s < p.num_seqs; ++s)
    if (enter_seq(p, c, s)) return;
  c.s = p.num_seqs;
}

// Warp-uniform window of 32 block-table entries of one sequence.
struct BtWindow {
  int s, lo, reg;
};

__device__ __forceinline__ int bt_lookup(const RowsParams& p, BtWindow& w, int s, int lb, int lane) {
  if (s != w.s || lb < w.lo || lb >= w.lo + 32) {
    w.s = s;
    w.lo = lb;
    const int idx = lb + lane;
    w.reg = idx < p.max_blocks ? __ldg(p.block_tables + static_cast<long long>(s) * p.max_blocks + idx) : -1;
  }
  return __shfl_sync(FULL_MASK, w.reg, lb - w.lo);
}

// First warp whose range [T*w/W, T*(w+1)/W) contains unit u.
__device__ __forceinline__ int owner_warp(long long u, long long T, long long W) {
  return static_cast<int>(((u + 1) * W + T - 1) / T - 1);
}

__device__ __forceinline__ long long range_start(long long w, long long T, long long W) { return T * w / W; }

template <int D, int NT>
struct RowsShape {
  static constexpr int KT = D / 16;                    // k-steps of QK^T, m-tiles of PV
  static constexpr int PIECES = D / 64;                // 64-column TMA boxes per row
  static constexpr int HALF_BYTES = TILE_KEYS * D * 2; // K (or V) bytes of a tile
  static constexpr int STAGE_BYTES = 2 * HALF_BYTES;
  static constexpr int SLOT_O = KT * NT * 32 * 4;      // O^T fragment floats of a partial
  static constexpr int SLOT_FLOATS = ((SLOT_O + 2 * NT * 8) + 63) / 64 * 64;
};

// Write normalised O for one segment: O^T fragments -> bf16 -> movmatrix -> rows of out.
template <int D, int NT>
__device__ __forceinline__ void store_output(const RowsParams& p, const float (&o)[D / 16][NT][4],
                                             const float (&l)[NT][2], int row, int kvh, int lane) {
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float inv0 = 1.f / l[nt][0], inv1 = 1.f / l[nt][1];
    const int head = nt * 8 + g;
    __nv_bfloat16* base = static_cast<__nv_bfloat16*>(p.out) +
                          (static_cast<long long>(row) * p.num_q_heads + kvh * p.group + head) * D + 2 * c;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      const uint32_t y0 = movmatrix_trans(pack_bf16x2(o[mt][nt][0] * inv0, o[mt][nt][1] * inv1));
      const uint32_t y1 = movmatrix_trans(pack_bf16x2(o[mt][nt][2] * inv0, o[mt][nt][3] * inv1));
      if (head < p.group) {
        *reinterpret_cast<uint32_t*>(base + 16 * mt) = y0;
        *reinterpret_cast<uint32_t*>(base + 16 * mt + 8) = y1;
      }
    }
  }
}

__device__ __forceinline__ void zero_rows(const RowsParams& p, int q0, int nrows, int head_dim) {
  uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                      static_cast<long long>(q0) * p.num_q_heads * head_dim);
  const long long n = static_cast<long long>(nrows) * p.num_q_heads * head_dim / 8;
  for (long long k = 0; k < n; ++k) o[k] = make_uint4(0, 0, 0, 0);
}

template <int D, int NT, int R>
__global__ void __launch_bounds__(ROWS_THREADS, 1)
    rows_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                const RowsParams p) {
  using S = RowsShape<D, NT>;
  constexpr int KT = S::KT;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[ROWS_WARPS][R];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gw = blockIdx.x * ROWS_WARPS + warp;
  const int g = lane >> 2, c = lane & 3;

  // ---- pass 1: total tile count; rows without a key are written as zeros
  long long T = 0;
  for (int base = 0; base < p.num_seqs; base += 32) {
    const int s = base + lane;
    long long u = 0;
    if (s < p.num_seqs) {
      const SeqInfo si = seq_info(p, s);
      u = seq_units(p, si);
      const int nzero = min(si.qlen, max(0, si.qlen - si.ctx));
      if (nzero > 0 && (s % p.total_warps) == gw) zero_rows(p, si.q0, nzero, D);
    }
    T += warp_sum64(u);
  }
  if (T == 0) return;
  const long long W = T < p.total_warps ? T : p.total_warps;
  if (gw >= W) return;
  const long long a = range_start(gw, T, W), e = range_start(gw + 1, T, W);
  const long long count = e - a;

  // ---- pass 2: the segment that holds unit a
  Cursor cc;
  {
    long long acc = 0;
    int s_found = -1;
    long long seq_base = 0;
    for (int base = 0; base < p.num_seqs && s_found < 0; base += 32) {
      const int s = base + lane;
      long long u = 0;
      if (s < p.num_seqs) u = seq_units(p, seq_info(p, s));
      const long long incl = warp_incl_scan64(u, lane);
      const long long chunk = __shfl_sync(FULL_MASK, incl, 31);
      if (acc + chunk > a) {
        const unsigned hit = __ballot_sync(FULL_MASK, acc + incl > a);
        const int src = __ffs(hit) - 1;
        s_found = base + src;
        seq_base = acc + __shfl_sync(FULL_MASK, incl - u, src);
      }
      acc += chunk;
    }
    const SeqInfo si = seq_info(p, s_found);
    cc.s = s_found;
    cc.qlen = si.qlen;
    cc.q0 = si.q0;
    cc.p0 = si.ctx - si.qlen;
    const int i0 = cc.p0 < 0 ? -cc.p0 : 0;
    const long long o = a - seq_base;
    const long long base_tiles = tiles_upto(cc.p0 + i0);
    int lo = i0, hi = si.qlen - 1;
    while (lo < hi) {  // last row whose first unit is <= o
      const int mid = (lo + hi + 1) >> 1;
      if (static_cast<long long>(p.num_kv_heads) * (tiles_upto(cc.p0 + mid) - base_tiles) <= o)
        lo = mid;
      else
        hi = mid - 1;
    }
    cc.i = lo;
    cc.nkeys = cc.p0 + lo + 1;
    cc.n = ceil16(cc.nkeys);
    const long long rem = o - static_cast<long long>(p.num_kv_heads) * (tiles_upto(cc.p0 + lo) - base_tiles);
    cc.h = static_cast<int>(rem / cc.n);
    cc.t = static_cast<int>(rem % cc.n);
    cc.u = a;
  }

  // ---- per-warp TMA ring
  uint8_t* ring = align1024(smem_raw) + static_cast<size_t>(warp) * R * S::STAGE_BYTES;
  uint64_t* bar = bars[warp];
  if (lane == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
#pragma unroll
    for (int k = 0; k < R; ++k) mbar_init(&bar[k], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = policy_evict_first();

  Cursor lc = cc;
  BtWindow win{-1, 0, -1};
  auto issue = [&](int stage) {
    const int key0 = lc.t * TILE_KEYS;
    const int lb = key0 / p.block_size, y = key0 - lb * p.block_size;
    const int blk = bt_lookup(p, win, lc.s, lb, lane);
    if (lane == 0) {
      if (blk < 0 || blk >= p.num_blocks) set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
      uint8_t* st = ring + stage * S::STAGE_BYTES;
      mbar_arrive_expect_tx(&bar[stage], S::STAGE_BYTES);
#pragma unroll
      for (int pc = 0; pc < S::PIECES; ++pc) {
        tma_load_4d(st + pc * 2048, &tmk, &bar[stage], pc * 64, y, lc.h, blk, pol);
        tma_load_4d(st + S::HALF_BYTES + pc * 2048, &tmv, &bar[stage], pc * 64, y, lc.h, blk, pol);
      }
    }
    advance(p, lc);
  };

  long long issued = 0;
  for (; issued < R && issued < count; ++issued) issue(static_cast<int>(issued));

  float o[KT][NT][4];
  uint32_t qb[NT][KT][2];
  float m[NT][2], l[NT][2];
  bool began = false;
  long long piece_j0 = 0;
  long long stopped_at = -1;

  for (long long j = 0; j < count; ++j) {
    const int stage = static_cast<int>(j % R);
    const uint32_t phase = static_cast<uint32_t>((j / R) & 1);

    if (j == 0 || cc.t == 0) {  // a piece starts: load the G query rows of this KV head
      began = (cc.t == 0);
      piece_j0 = j;
      const int row = cc.q0 + cc.i;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int head = nt * 8 + g;
        const bool ok = head < p.group;
        const uint32_t* qp = reinterpret_cast<const uint32_t*>(
            static_cast<const __nv_bfloat16*>(p.q) +
            (static_cast<long long>(row) * p.num_q_heads + cc.h * p.group + (ok ? head : 0)) * D);
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
          qb[nt][kk][0] = ok ? __ldg(qp + 8 * kk + c) : 0u;
          qb[nt][kk][1] = ok ? __ldg(qp + 8 * kk + 4 + c) : 0u;
        }
        m[nt][0] = m[nt][1] = -INFINITY;
        l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
        for (int mt = 0; mt < KT; ++mt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
      }
    }

    if (!mbar_wait(&bar[stage], phase)) {
      set_status(p.status, PA_STATUS_BIT(PA_ERR_TIMEOUT));
      stopped_at = j;
      break;
    }
    uint8_t* kt = ring + stage * S::STAGE_BYTES;
    uint8_t* vt = kt + S::HALF_BYTES;
    const int nvalid = min(TILE_KEYS, cc.nkeys - cc.t * TILE_KEYS);
    if (nvalid < TILE_KEYS) {  // rows past the context may hold anything: zero V there
      const int nz = (TILE_KEYS - nvalid) * S::PIECES * 8;
      for (int k = lane; k < nz; k += 32) {
        const int r = nvalid + k / (S::PIECES * 8);
        const int rest = k % (S::PIECES * 8);
        *reinterpret_cast<uint4*>(vt + (rest >> 3) * 2048 + r * 128 + (rest & 7) * 16) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }

    // S^T[key, head] = K . Q^T
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
    {
      const int mi = lane >> 3;
      const int r = (lane & 7) + (mi & 1) * 8;
      const uint32_t kbase = smem_u32(kt);
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kbase + (kk >> 2) * 2048 + sw128(r, 2 * (kk & 3) + (mi >> 1)), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(sacc[nt], a0, a1, a2, a3, qb[nt][kk][0], qb[nt][kk][1]);
      }
    }

    // online softmax on the fragment: this lane holds keys g, g+8 of heads 2c, 2c+1
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float s0 = sacc[nt][0] * p.scale_log2, s1 = sacc[nt][1] * p.scale_log2;
      float s2 = sacc[nt][2] * p.scale_log2, s3 = sacc[nt][3] * p.scale_log2;
      if (g >= nvalid) s0 = s1 = -INFINITY;
      if (g + 8 >= nvalid) s2 = s3 = -INFINITY;
      float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(FULL_MASK, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(FULL_MASK, mx1, off));
      }
      const float mn0 = fmaxf(m[nt][0], mx0), mn1 = fmaxf(m[nt][1], mx1);
      const float al0 = fast_exp2(m[nt][0] - mn0), al1 = fast_exp2(m[nt][1] - mn1);
      m[nt][0] = mn0;
      m[nt][1] = mn1;
      const float p0 = fast_exp2(s0 - mn0), p2 = fast_exp2(s2 - mn0);
      const float p1 = fast_exp2(s1 - mn1), p3 = fast_exp2(s3 - mn1);
      l[nt][0] = l[nt][0] * al0 + p0 + p2;
      l[nt][1] = l[nt][1] * al1 + p1 + p3;
#pragma unroll
      for (int mt = 0; mt < KT; ++mt) {
        o[mt][nt][0] *= al0;
        o[mt][nt][1] *= al1;
        o[mt][nt][2] *= al0;
        o[mt][nt][3] *= al1;
      }
      pb[nt][0] = movmatrix_trans(pack_bf16x2(p0, p1));
      pb[nt][1] = movmatrix_trans(pack_bf16x2(p2, p3));
    }

    // O^T[d, head] += V^T . P^T
    {
      const int mi = lane >> 3;
      const int r = (lane & 7) + (mi >> 1) * 8;
      const uint32_t vbase = smem_u32(vt);
#pragma unroll
      for (int mt = 0; mt < KT; ++mt) {
        const int cg = 2 * mt + (mi & 1);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_trans(vbase + (cg >> 3) * 2048 + sw128(r, cg & 7), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
      }
    }

    // refill this stage
    __syncwarp();
    if (issued < count) {
      if (lane == 0) fence_proxy_async_smem();
      issue(stage);
      ++issued;
    }

    // ---- end of a piece: write the output or a partial
    if (j == count - 1 || cc.t == cc.n - 1) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          float v = l[nt][q2];
          v += __shfl_xor_sync(FULL_MASK, v, 4);
          v += __shfl_xor_sync(FULL_MASK, v, 8);
          v += __shfl_xor_sync(FULL_MASK, v, 16);
          l[nt][q2] = v;
        }
      const int row = cc.q0 + cc.i;
      if (began && cc.t == cc.n - 1) {
        store_output<D, NT>(p, o, l, row, cc.h, lane);
      } else {
        const int slot = 2 * gw + (piece_j0 == 0 ? 0 : 1);
        float* ps = p.partials + static_cast<long long>(slot) * S::SLOT_FLOATS;
#pragma unroll
        for (int mt = 0; mt < KT; ++mt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            reinterpret_cast<float4*>(ps)[(mt * NT + nt) * 32 + lane] =
                make_float4(o[mt][nt][0], o[mt][nt][1], o[mt][nt][2], o[mt][nt][3]);
        if (lane < 4) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            ps[S::SLOT_O + nt * 8 + 2 * lane] = m[nt][0];
            ps[S::SLOT_O + nt * 8 + 2 * lane + 1] = m[nt][1];
            ps[S::SLOT_O + NT * 8 + nt * 8 + 2 * lane] = l[nt][0];
            ps[S::SLOT_O + NT * 8 + nt * 8 + 2 * lane + 1] = l[nt][1];
          }
        }
        __threadfence();
        __syncwarp();
        const long long segA = cc.u - cc.t, segB = segA + cc.n;
        const int w0 = owner_warp(segA, T, W), w1 = owner_warp(segB - 1, T, W);
        const int npieces = w1 - w0 + 1;
        int* counter = p.counters + static_cast<long long>(row) * p.num_kv_heads + cc.h;
        int old = 0;
        if (lane == 0) old = atomicAdd(counter, 1);
        old = __shfl_sync(FULL_MASK, old, 0);
        if (old == npieces - 1) {  // last arrival merges every piece of the segment
          __threadfence();
          float mm[NT][2], acc[KT][NT][4], ll[NT][2];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mm[nt][0] = mm[nt][1] = -INFINITY;
            ll[nt][0] = ll[nt][1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < KT; ++mt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
          }
          for (int k = 0; k < npieces; ++k) {
            const int wk = w0 + k;
            const int sk = 2 * wk + ((k == 0 && range_start(wk, T, W) < segA) ? 1 : 0);
            const float* pk = p.partials + static_cast<long long>(sk) * S::SLOT_FLOATS;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mm[nt][0] = fmaxf(mm[nt][0], __ldcg(pk + S::SLOT_O + nt * 8 + 2 * c));
              mm[nt][1] = fmaxf(mm[nt][1], __ldcg(pk + S::SLOT_O + nt * 8 + 2 * c + 1));
            }
          }
          for (int k = 0; k < npieces; ++k) {
            const int wk = w0 + k;
            const int sk = 2 * wk + ((k == 0 && range_start(wk, T, W) < segA) ? 1 : 0);
            const float* pk = p.partials + static_cast<long long>(sk) * S::SLOT_FLOATS;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const float f0 = fast_exp2(__ldcg(pk + S::SLOT_O + nt * 8 + 2 * c) - mm[nt][0]);
              const float f1 = fast_exp2(__ldcg(pk + S::SLOT_O + nt * 8 + 2 * c + 1) - mm[nt][1]);
              ll[nt][0] += f0 * __ldcg(pk + S::SLOT_O + NT * 8 + nt * 8 + 2 * c);
              ll[nt][1] += f1 * __ldcg(pk + S::SLOT_O + NT * 8 + nt * 8 + 2 * c + 1);
#pragma unroll
              for (int mt = 0; mt < KT; ++mt) {
                const float4 v = __ldcg(reinterpret_cast<const float4*>(pk) + (mt * NT + nt) * 32 + lane);
                acc[mt][nt][0] += f0 * v.x;
                acc[mt][nt][1] += f1 * v.y;
                acc[mt][nt][2] += f0 * v.z;
                acc[mt][nt][3] += f1 * v.w;
              }
            }
          }
          store_output<D, NT>(p, acc, ll, row, cc.h, lane);
          if (lane == 0) *counter = 0;  // leave the workspace zeroed for the next call
        }
      }
    }
    advance(p, cc);
  }

  if (stopped_at >= 0) {  // let copies still in flight land before the shared memory goes away
    for (long long j = stopped_at + 1; j < issued; ++j) mbar_wait(&bar[j % R], static_cast<uint32_t>((j / R) & 1));
  }
}

// ------------------------------------------------------------------ host side

template <int D, int NT, int R>
static int launch_rows_t(const RowsParams& p0, const CUtensorMap& tmk, const CUtensorMap& tmv, cudaStream_t stream,
                         int num_sms) {
  using S = RowsShape<D, NT>;
  const int smem = ROWS_WARPS * R * S::STAGE_BYTES + 1024;
  auto kern = rows_kernel<D, NT, R>;
  static int configured_dev = -1;
  static int blocks_per_sm = 1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (configured_dev != dev) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return PA_ERR_CUDA;
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, ROWS_THREADS, smem) != cudaSuccess || nb < 1)
      return PA_ERR_CUDA;
    blocks_per_sm = nb > 2 ? 2 : nb;
    configured_dev = dev;
  }
  RowsParams p = p0;
  const int grid = num_sms * blocks_per_sm;
  p.total_warps = grid * ROWS_WARPS;
  kern<<<grid, ROWS_THREADS, smem, stream>>>(tmk, tmv, p);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int rows_supported(int group, int head_dim) {
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return 0;
  if (group < 1) return 0;
  if (head_dim == 256) return group <= 8;
  return group <= 16;
}

size_t rows_partials_bytes(int num_q_heads, int num_kv_heads, int head_dim, int num_sms) {
  const int group = num_q_heads / num_kv_heads;
  const int nt = group > 8 ? 2 : 1;
  const size_t o = static_cast<size_t>(head_dim / 16) * nt * 32 * 4;
  const size_t slot = (o + 2 * nt * 8 + 63) / 64 * 64;
  const size_t max_warps = static_cast<size_t>(num_sms) * 2 * ROWS_WARPS;
  return 2 * max_warps * slot * sizeof(float);
}

int launch_rows(const RowsParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, int head_dim,
                cudaStream_t stream, int num_sms) {
  const bool two = p.group > 8;
  switch (head_dim) {
    case 64:
      return two ? launch_rows_t<64, 2, 8>(p, tmk, tmv, stream, num_sms)
                 : launch_rows_t<64, 1, 8>(p, tmk, tmv, stream, num_sms);
    case 128:
      return two ? launch_rows_t<128, 2, 3>(p, tmk, tmv, stream, num_sms)
                 : launch_rows_t<128, 1, 3>(p, tmk, tmv, stream, num_sms);
    case 256:
      return launch_rows_t<256, 1, 3>(p, tmk, tmv, stream, num_sms);
    default:
      return PA_ERR_UNSUPPORTED;
  }
}

}  // namespace pa
