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
//  * Work unit = one 16-key tile (32 keys in the E4M3 kernel at head_dim 128
//    with one head tile) of one (query row, KV head) "segment".  All
//    G = Hq / Hkv query heads of the KV head ride along, so each K/V byte is
//    read from HBM once per step.  Each CTA scans context_lens into shared
//    memory (tile prefix sums per sequence), every warp takes an equal
//    contiguous range of the batch's T tiles: the split is exact to one tile
//    whatever the length mix, deterministic, and needs no host-side plan.
//  * A segment cut by a range boundary is finished as partial (m, l, O)
//    results, written with plain stores and recorded in a per-unit piece
//    table; after a grid barrier (cooperative launch) the pieces of every cut
//    segment are merged in order.  At most two partial slots per warp, no
//    second launch, no atomics on the streaming path.
//  * Tiles stream HBM -> shared memory through TMA (one 5-D box per K or V
//    tile of one (block, head), block ID as a coordinate, 128-byte swizzle),
//    a ring of R stages per warp completed on mbarriers.  Each warp is its own
//    producer and consumer and hands a stage back as soon as the tile is in
//    registers.
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

constexpr int TILE_KEYS = 16;  // keys per work unit, and per TMA box; a variant may take two boxes per unit
constexpr int ROWS_WARPS = 4;       // warps per CTA of the usual launch (2 or 3 CTAs per SM)
constexpr int ROWS_WARPS_WIDE = 8;  // warps per CTA when a CTA holds a whole SM (a launch on part of the GPU)
constexpr int ROWS_SLOTS_PER_WARP = 2;  // a warp's range cuts at most its first and its last segment
constexpr int ROWS_SMEM_SEQS = ROWS_SMEM_SEQS_HOST;  // sequences whose tile prefix sums live in shared memory
constexpr int ROWS_MAX_CTAS_PER_SM = 3;  // the workspace holds partial slots for this many CTAs per SM
// Accumulation chains of S = K Q^T per tile (bf16 path): 1, or 2 (even and odd k-steps).
#ifndef PA_ROWS_S_CHAINS
#define PA_ROWS_S_CHAINS 1
#endif
constexpr int ROWS_S_CHAINS = PA_ROWS_S_CHAINS;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// Work units (tiles of 2^tile_shift keys) of a segment with n keys.
__device__ __forceinline__ int ceil_tiles(const RowsParams& p, int n) {
  return (n + (1 << p.tile_shift) - 1) >> p.tile_shift;
}

// sum_{k=1}^{n} ceil(k / TK), TK = 2^tile_shift: tiles of the rows whose key counts are 1..n.
__device__ __forceinline__ long long tiles_upto(const RowsParams& p, int n) {
  if (n <= 0) return 0;
  const int sh = p.tile_shift;
  const long long tk = 1ll << sh, q = n >> sh, r = n & (tk - 1);
  return tk * q * (q + 1) / 2 + r * (q + 1);
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
  int ctx, qlen, q0;  // ctx: keys this kernel attends to, from key k0 on
  int k0;             // keys before k0 came from the shared-prefix pass
};

// First key this kernel attends to for sequence s: the shared-prefix span of
// its group, if it belongs to one (binary search over the group boundaries).
__device__ __forceinline__ int cascade_key0(const RowsParams& p, int s) {
  if (p.num_groups <= 0 || s < __ldg(p.group_start) || s >= __ldg(p.group_start + p.num_groups)) return 0;
  int lo = 0, hi = p.num_groups - 1;  // last g with group_start[g] <= s
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.group_start + mid) <= s)
      lo = mid;
    else
      hi = mid - 1;
  }
  return cascade_span(__ldg(p.group_prefix + lo));
}

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
  si.k0 = 0;
  if (p.num_groups > 0) {
    const int k0 = cascade_key0(p, s);
    if (k0 > 0 && si.qlen == 1 && si.ctx > k0) {
      si.k0 = k0;
      si.ctx -= k0;
    } else if (k0 > 0) {  // the newest token must lie after the shared prefix
      set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
    }
  }
  return si;
}

// Tiles of all (row, KV head) segments of one sequence.
__device__ __forceinline__ long long seq_units(const RowsParams& p, const SeqInfo& si) {
  if (p.skip_multi && si.qlen > 1) return 0;
  const int p0 = si.ctx - si.qlen;
  return static_cast<long long>(p.num_kv_heads) * (tiles_upto(p, si.ctx) - tiles_upto(p, p0 < 0 ? 0 : p0));
}

struct Cursor {
  int s, i, h, t;  // sequence, row within it, KV head, tile within the segment
  int n, nkeys;    // tiles and keys of the current segment
  int p0, qlen, q0;
  int k0;          // first key of the segments (after a shared prefix handled elsewhere)
  long long u;     // global unit index
};

__device__ __forceinline__ bool enter_seq(const RowsParams& p, Cursor& c, int s) {
  const SeqInfo si = seq_info(p, s);
  if (seq_units(p, si) == 0) return false;
  c.s = s;
  c.qlen = si.qlen;
  c.q0 = si.q0;
  c.k0 = si.k0;
  c.p0 = si.ctx - si.qlen;
  c.i = c.p0 < 0 ? -c.p0 : 0;  // first row that has a key
  c.h = 0;
  c.t = 0;
  c.nkeys = c.p0 + c.i + 1;
  c.n = ceil_tiles(p, c.nkeys);
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
    c.n = ceil_tiles(p, c.nkeys);
    return;
  }
  for (int s = c.s + 1; s < p.num_seqs; ++s)
    if (enter_seq(p, c, s)) return;
  c.s = p.num_seqs;
}

// Warp-uniform window of 128 block-table entries of one sequence (4 per lane).
struct BtWindow {
  int s, lo;
  int r[4];
};

__device__ __forceinline__ int bt_lookup(const RowsParams& p, BtWindow& w, int s, int lb, int lane) {
  if (s != w.s || lb < w.lo || lb >= w.lo + 128) {
    w.s = s;
    w.lo = lb;
    const int32_t* row = p.block_tables + static_cast<long long>(s) * p.max_blocks;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int idx = lb + 32 * k + lane;
      w.r[k] = idx < p.max_blocks ? __ldg(row + idx) : -1;
    }
  }
  const int e = lb - w.lo, k = e >> 5;
  const int v = k == 0 ? w.r[0] : k == 1 ? w.r[1] : k == 2 ? w.r[2] : w.r[3];
  return __shfl_sync(FULL_MASK, v, e & 31);
}

__device__ __forceinline__ long long range_start(long long w, long long T, long long W) { return T * w / W; }

template <int D, int NT, bool F8 = false, int TK = TILE_KEYS>
struct RowsShape {
  static constexpr int KT = D / 16;                    // k-steps of QK^T, m-tiles of PV
  static constexpr int BOX_BYTES = TILE_KEYS * D * (F8 ? 1 : 2);  // one TMA box: 16 rows of one (block, head)
  static constexpr int HALF_BYTES = TK * D * (F8 ? 1 : 2);        // K (or V) bytes of a tile
  static constexpr int STAGE_BYTES = 2 * HALF_BYTES;
  static constexpr int SLOT_O = KT * NT * 32 * 4;      // O^T fragment floats of a partial
  static constexpr int SLOT_M = SLOT_O;                // running maxima (8 NT floats)
  static constexpr int SLOT_L = SLOT_O + 8 * NT;       // sums (8 NT floats)
  static constexpr int SLOT_NEXT = SLOT_O + 16 * NT;   // next slot of the segment + 1 (int), 0 = end
  static constexpr int SLOT_FLOATS = (SLOT_NEXT + 1 + 63) / 64 * 64;
};

// Write normalised O for one segment: O^T fragments -> bf16 -> movmatrix -> rows of out.
// FP8 caches: the accumulator rows g and g + 8 of m-tile mt are head-dim
// 16 mt + 2g and 16 mt + 2g + 1 (the order the E4M3 V fragments are built in),
// so each lane stores its two heads' pairs directly; O also takes the V scale.
template <int D, int NT, bool F8 = false>
__device__ __forceinline__ void store_output(const RowsParams& p, const float (&o)[D / 16][NT][4],
                                             const float (&l)[NT][2], int row, int kvh, int lane) {
  const int g = lane >> 2, c = lane & 3;
  if constexpr (F8) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int head = nt * 8 + 2 * c + e;
        const float inv = p.v_scale / l[nt][e];
        __nv_bfloat16* base = static_cast<__nv_bfloat16*>(p.out) +
                              (static_cast<long long>(row) * p.num_q_heads + kvh * p.group + head) * D + 2 * g;
        if (head < p.group) {
#pragma unroll
          for (int mt = 0; mt < D / 16; ++mt)
            *reinterpret_cast<uint32_t*>(base + 16 * mt) = pack_bf16x2(o[mt][nt][e] * inv, o[mt][nt][2 + e] * inv);
        }
      }
    return;
  }
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

// Position a cursor on global unit a (a < T).  The sequence comes from the
// shared-memory prefix of per-sequence tile counts when there is one (binary
// search), else from a scan of context_lens; the row from a binary search
// over the closed-form tile counts of its rows.
__device__ __forceinline__ void seek(const RowsParams& p, const long long* pfx, long long a, int lane, Cursor& cc) {
  int s_found = -1;
  long long seq_base = 0;
  if (pfx) {
    int lo = 0, hi = p.num_seqs;  // first k with pfx[k] > a, minus one
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (pfx[mid + 1] > a)
        hi = mid;
      else
        lo = mid + 1;
    }
    s_found = lo;
    seq_base = pfx[lo];
  } else {
    long long acc = 0;
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
  }
  const SeqInfo si = seq_info(p, s_found);
  cc.s = s_found;
  cc.qlen = si.qlen;
  cc.q0 = si.q0;
  cc.k0 = si.k0;
  cc.p0 = si.ctx - si.qlen;
  const int i0 = cc.p0 < 0 ? -cc.p0 : 0;
  const long long o = a - seq_base;
  const long long base_tiles = tiles_upto(p, cc.p0 + i0);
  int lo = i0, hi = si.qlen - 1;
  while (lo < hi) {  // last row whose first unit is <= o
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<long long>(p.num_kv_heads) * (tiles_upto(p, cc.p0 + mid) - base_tiles) <= o)
      lo = mid;
    else
      hi = mid - 1;
  }
  cc.i = lo;
  cc.nkeys = cc.p0 + lo + 1;
  cc.n = ceil_tiles(p, cc.nkeys);
  const long long rem = o - static_cast<long long>(p.num_kv_heads) * (tiles_upto(p, cc.p0 + lo) - base_tiles);
  cc.h = static_cast<int>(rem / cc.n);
  cc.t = static_cast<int>(rem % cc.n);
  cc.u = a;
}

// Fold the shared-prefix partials of (sequence seq, KV head kvh) into the state
// of its segment: per query head, with m' = max(m, max over the slices k of m_k),
// O <- O e^(m - m') + sum_k O_k e^(m_k - m'), l likewise.  `slices` is a bit
// mask over the records 0 .. CASCADE_SPLITS; all its records load at once
// (maxima and sums first, then the O rows), not one slice after another.
template <int D, int NT>
__device__ __forceinline__ void fold_prefix(const RowsParams& p, unsigned slices, float (&o)[D / 16][NT][4],
                                            float (&m)[NT][2], float (&l)[NT][2], int seq, int kvh, int lane) {
  constexpr int NREC = CASCADE_SPLITS + 1;
  constexpr int REC = cascade_record_floats(D);
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int head = nt * 8 + 2 * c + e;
      if (head >= p.group) continue;
      const float* base = p.casc_partials +
                          (static_cast<long long>(seq) * p.num_q_heads + kvh * p.group + head) * NREC * REC;
      float mk[NREC], w[NREC];
      float mn = m[nt][e];
#pragma unroll
      for (int k = 0; k < NREC; ++k) {
        mk[k] = (slices >> k) & 1 ? __ldcg(base + k * REC + D) : -INFINITY;
        mn = fmaxf(mn, mk[k]);
      }
      const float f = fast_exp2(m[nt][e] - mn);
      float lt = l[nt][e] * f;
#pragma unroll
      for (int k = 0; k < NREC; ++k) {
        w[k] = (slices >> k) & 1 ? fast_exp2(mk[k] - mn) : 0.f;
        if ((slices >> k) & 1) lt += w[k] * __ldcg(base + k * REC + D + 1);
      }
      m[nt][e] = mn;
      l[nt][e] = lt;
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {  // accumulator rows: head dim 16 mt + g and 16 mt + g + 8
        float a = o[mt][nt][e] * f, b = o[mt][nt][2 + e] * f;
#pragma unroll
        for (int k = 0; k < NREC; ++k)
          if ((slices >> k) & 1) {
            a += w[k] * __ldcg(base + k * REC + 16 * mt + g);
            b += w[k] * __ldcg(base + k * REC + 16 * mt + g + 8);
          }
        o[mt][nt][e] = a;
        o[mt][nt][2 + e] = b;
      }
    }
}

// Store the unnormalised state of a whole private segment in the shared-prefix
// buffer's last slot (index CASCADE_SPLITS), row-major per query head.
template <int D, int NT>
__device__ __forceinline__ void store_own_partial(const RowsParams& p, const float (&o)[D / 16][NT][4],
                                                  const float (&m)[NT][2], const float (&l)[NT][2], int seq, int kvh,
                                                  int lane) {
  const int g = lane >> 2, c = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int head = nt * 8 + 2 * c + e;
      if (head >= p.group) continue;
      float* dst = const_cast<float*>(p.casc_partials) +
                   ((static_cast<long long>(seq) * p.num_q_heads + kvh * p.group + head) * (CASCADE_SPLITS + 1) +
                    CASCADE_SPLITS) * cascade_record_floats(D);
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        dst[16 * mt + g] = o[mt][nt][e];
        dst[16 * mt + g + 8] = o[mt][nt][2 + e];
      }
      if (g == 0) {
        dst[D] = m[nt][e];
        dst[D + 1] = l[nt][e];
      }
    }
}

// Merge the partial (m, l, O) results of the pieces of segment [segA, segA + n)
// and write the normalised output row.  Piece k recorded (slot, tiles) at the
// table entry of its first unit, so the walk visits the pieces in order; one
// pass with a running maximum.
template <int D, int NT, bool F8>
__device__ __forceinline__ void merge_segment(const RowsParams& p, long long segA, int n, int row, int kvh, int lane) {
  using S = RowsShape<D, NT, F8>;
  constexpr int KT = S::KT;
  const int c = lane & 3;
  float mm[NT][2], acc[KT][NT][4], ll[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    mm[nt][0] = mm[nt][1] = -INFINITY;
    ll[nt][0] = ll[nt][1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < KT; ++mt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
  }
  for (int t = 0; t < n;) {
    const long long e = __ldcg(p.table + segA + t);
    const int slot = static_cast<int>(e & 0xffffffffll), tiles = static_cast<int>(e >> 32);
    if (tiles <= 0 || slot < 0) {  // cannot happen when every piece recorded itself
      set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
      break;
    }
    t += tiles;
    const float* pk = p.partials + static_cast<long long>(slot) * S::SLOT_FLOATS;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float f[2], gk[2];
#pragma unroll
      for (int e2 = 0; e2 < 2; ++e2) {
        const float mk = __ldcg(pk + S::SLOT_M + nt * 8 + 2 * c + e2);
        const float mn = fmaxf(mm[nt][e2], mk);
        f[e2] = fast_exp2(mm[nt][e2] - mn);  // rescales what was merged so far
        gk[e2] = fast_exp2(mk - mn);         // weight of this piece
        mm[nt][e2] = mn;
        ll[nt][e2] = ll[nt][e2] * f[e2] + gk[e2] * __ldcg(pk + S::SLOT_L + nt * 8 + 2 * c + e2);
      }
#pragma unroll
      for (int mt = 0; mt < KT; ++mt) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(pk) + (mt * NT + nt) * 32 + lane);
        acc[mt][nt][0] = acc[mt][nt][0] * f[0] + gk[0] * v.x;
        acc[mt][nt][1] = acc[mt][nt][1] * f[1] + gk[1] * v.y;
        acc[mt][nt][2] = acc[mt][nt][2] * f[0] + gk[0] * v.z;
        acc[mt][nt][3] = acc[mt][nt][3] * f[1] + gk[1] * v.w;
      }
    }
  }
  if (p.num_groups > 0) {
    const int span = seq_info(p, row).k0;  // decode: row = sequence; 0 if its keys were not split
    if (span > 0) {
      // the prefix slices, and with n == 0 the private part too (one piece, kept in the last slot)
      const unsigned slices = ((1u << cascade_splits(span)) - 1u) | (n == 0 ? 1u << CASCADE_SPLITS : 0u);
      fold_prefix<D, NT>(p, slices, acc, mm, ll, row, kvh, lane);
    }
  }
  store_output<D, NT, F8>(p, acc, ll, row, kvh, lane);
}

// 8 bf16 (one 16-byte vector) -> 8 E4M3 codes of value * inv_scale (the
// product in binary32, then nearest-even with saturation).
__device__ __forceinline__ uint32_t bf16x2_bits_to_e4m3x2(uint32_t w, float inv) {
  const float lo = __uint_as_float(w << 16) * inv, hi = __uint_as_float(w & 0xffff0000u) * inv;
  return f32x2_to_e4m3x2(lo, hi);
}
__device__ __forceinline__ uint2 quantize8(uint4 x, float inv) {
  return make_uint2(bf16x2_bits_to_e4m3x2(x.x, inv) | (bf16x2_bits_to_e4m3x2(x.y, inv) << 16),
                    bf16x2_bits_to_e4m3x2(x.z, inv) | (bf16x2_bits_to_e4m3x2(x.w, inv) << 16));
}

// Fused cache append (decode): write row s of k_new / v_new, sequence s's
// newest token, to position context_lens[s] - 1 of its block table, every KV
// head, 16-byte vectors over the whole grid.  The attention does not read
// these bytes back (it takes the newest key from k_new / v_new), so nothing
// waits for the stores.
template <int D, bool F8>
__device__ __forceinline__ void fused_append(const RowsParams& p, long long tid, long long nthreads) {
  constexpr int VEC = D / 8;  // 16-byte vectors of a bf16 row
  const long long n = static_cast<long long>(p.num_seqs) * p.num_kv_heads * VEC;
  for (long long i = tid; i < n; i += nthreads) {
    const int v = static_cast<int>(i % VEC);
    const long long sh = i / VEC;
    const int h = static_cast<int>(sh % p.num_kv_heads), s = static_cast<int>(sh / p.num_kv_heads);
    const int ctx = __ldg(p.context_lens + s);
    if (ctx < 1) continue;
    const int pos = ctx - 1, lb = pos / p.block_size;
    if (lb >= p.max_blocks) continue;  // reported by the attention's own length check
    const int blk = __ldg(p.block_tables + static_cast<long long>(s) * p.max_blocks + lb);
    if (blk < 0 || blk >= p.num_blocks) {
      set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
      continue;
    }
    const long long src = sh * VEC + v;
    const long long dst = ((static_cast<long long>(blk) * p.num_kv_heads + h) * p.block_size + pos % p.block_size) *
                              VEC + v;
    const uint4 kx = __ldg(reinterpret_cast<const uint4*>(p.k_new) + src);
    const uint4 vx = __ldg(reinterpret_cast<const uint4*>(p.v_new) + src);
    if constexpr (F8) {  // 8 bf16 -> 8 E4M3 codes of value / scale (8 bytes)
      reinterpret_cast<uint2*>(p.k_cache)[dst] = quantize8(kx, p.k_inv_scale);
      reinterpret_cast<uint2*>(p.v_cache)[dst] = quantize8(vx, p.v_inv_scale);
    } else {
      reinterpret_cast<uint4*>(p.k_cache)[dst] = kx;
      reinterpret_cast<uint4*>(p.v_cache)[dst] = vx;
    }
  }
}

// What the consumer needs to know about the tile in a ring stage; written by
// the issuing lane before the TMA, read by the warp after the stage completes.
struct TileMeta {
  long long u;  // global unit index
  int row, h, t, n, nkeys;
  int flags;  // bit 0: first tile of this warp's range, bit 1: last tile of it
};

// CTAs per SM a variant is compiled for: the E4M3 kernel with one head tile
// and 16-key tiles is bound by instruction latency (the code conversions), so
// it runs three CTAs per SM (12 warps) in at most 168 registers; the others
// run two.
template <int D, int NT, bool F8, int TK>
constexpr int rows_ctas_per_sm() {
  return (F8 && D == 128 && NT == 1 && TK == 16) ? 3 : 2;
}

// TK: keys per work unit and ring stage, 16 or 32.  With 32 (the E4M3 kernel
// at head_dim 128 with one head tile) a stage holds two 16-row TMA boxes per
// K and V and the warp takes two 16-key m-tiles per softmax step, so the
// per-tile bookkeeping covers twice the bytes.
template <int D, int NT, int R, bool F8, int TK, int NW>
__global__ void __launch_bounds__(NW * 32, rows_ctas_per_sm<D, NT, F8, TK>() == 3 ? 3 : 1)
    rows_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                const __grid_constant__ RowsParams p) {
  static_assert(TK == TILE_KEYS || (TK == 2 * TILE_KEYS && F8 && D == 128 && NT == 1), "32-key tiles: E4M3, D 128, G <= 8");
  using S = RowsShape<D, NT, F8, TK>;
  constexpr int KT = S::KT;
  extern __shared__ uint8_t smem_raw[];
  constexpr int ROWS_THREADS = NW * 32;
  __shared__ __align__(8) uint64_t bars[NW][R];
  __shared__ TileMeta metas[NW][R];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gw = blockIdx.x * NW + warp;
  const int g = lane >> 2, c = lane & 3;
  uint8_t* base = align1024(smem_raw);
  const bool use_pfx = p.num_seqs <= ROWS_SMEM_SEQS;
  long long* pfx = use_pfx ? reinterpret_cast<long long*>(base + NW * R * S::STAGE_BYTES) : nullptr;

  // Split by SM rate: this CTA's SM, registered at once so that the atomics'
  // round trips overlap the prologue (their results are read after it).
  const bool partial = p.weighted && static_cast<int>(gridDim.x) < p.num_sms;  // one CTA on each of some SMs
  unsigned sm_id = 0;
  int sm_claim = 0;
  if (p.weighted && threadIdx.x == 0) {
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm_id));
    if (sm_id < static_cast<unsigned>(p.num_sms)) {
      if (partial) {
        atomicOr(p.sm_mask + (sm_id >> 5), 1u << (sm_id & 31));
        __threadfence();
        atomicAdd(p.sched + 2, 1);
      } else {
        sm_claim = atomicAdd(p.sm_slots + sm_id, 1);  // which of the SM's CTAs this one is
      }
    }
  }

  // ---- prologue: tiles of every sequence, their prefix sums, the total T.
  // Rows without a key are written as zeros here (each by one thread).
  long long T = 0;
  if (use_pfx) {
    for (int s = threadIdx.x; s < p.num_seqs; s += ROWS_THREADS) pfx[s + 1] = seq_units(p, seq_info(p, s));
    if (threadIdx.x == 0) pfx[0] = 0;
    __syncthreads();
    if (warp == 0) {
      long long carry = 0;
      for (int b0 = 0; b0 < p.num_seqs; b0 += 32) {
        const int s = b0 + lane;
        const long long v = s < p.num_seqs ? pfx[s + 1] : 0;
        const long long incl = warp_incl_scan64(v, lane);
        if (s < p.num_seqs) pfx[s + 1] = carry + incl;
        carry += __shfl_sync(FULL_MASK, incl, 31);
      }
    }
    __syncthreads();
    T = pfx[p.num_seqs];
  } else {
    for (int b0 = 0; b0 < p.num_seqs; b0 += 32) {
      const int s = b0 + lane;
      T += warp_sum64(s < p.num_seqs ? seq_units(p, seq_info(p, s)) : 0);
    }
  }

  // Everything above reads only the batch metadata.  From here on the kernel
  // reads the cache (which the append kernel before it may still be writing)
  // and writes out: wait for the grids this launch depends on.
  grid_dependency_wait();
  // beside the chunk kernel: the append is visible now, so that kernel may
  // take the SMs this launch leaves free
  if (p.trigger_early) grid_launch_dependents();
  for (int s = blockIdx.x * ROWS_THREADS + threadIdx.x; s < p.num_seqs; s += gridDim.x * ROWS_THREADS) {
    const SeqInfo si = seq_info(p, s);  // rows without a key are written as zeros
    const int nzero = min(si.qlen, max(0, si.qlen - si.ctx));
    if (nzero > 0) zero_rows(p, si.q0, nzero, D);
  }
  if (T > p.table_len) {  // the host sized the piece table for the largest possible batch
    set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
    T = 0;
  }

  // ---- this warp's contiguous range [a, e) of the T units, and its index r
  // among the ranges (its partial-result slots are 2r and 2r + 1)
  long long ra = 0, re = 0;
  int r_index = gw;
  if (p.weighted && T > 0) {
    // each SM takes a share of the units in proportion to its rate, cut
    // equally between the warps of its CTAs; which CTA of an SM takes which
    // part is decided by arrival (the parts, hence the result, do not depend
    // on it)
    __shared__ int sm_local, sm_ok;
    __shared__ long long sm_lo, sm_all;
    if (threadIdx.x == 0) {
      const unsigned smid = sm_id;
      sm_ok = smid < static_cast<unsigned>(p.num_sms);
      if (partial && sm_ok) {  // wait (bounded) until every CTA has registered its SM
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(p.sched + 2) < static_cast<int>(gridDim.x)) {
          if (globaltimer_ns() - t0 > WAIT_NS) {
            set_status(p.status, PA_STATUS_BIT(PA_ERR_TIMEOUT));
            sm_ok = 0;
            break;
          }
          __nanosleep(64);
        }
      }
      sm_local = (partial ? 0 : sm_claim) * 65536 + static_cast<int>(smid);  // (local index, SM id)
      if (!partial && sm_ok) {  // a whole-GPU launch: the host's prefix sums
        sm_lo = p.sm_prefix[smid];
        sm_all = p.sm_prefix[p.num_sms];
      }
    }
    if (partial) {  // the rates of the registered SMs only: a reduction over the CTA's threads
      __syncthreads();
      const unsigned me = static_cast<unsigned>(sm_local & 65535);
      long long lo = 0, all = 0;
      for (int q = threadIdx.x; q < p.num_sms; q += ROWS_THREADS) {
        if (!((__ldcg(p.sm_mask + (q >> 5)) >> (q & 31)) & 1u)) continue;
        all += p.sm_rate[q];
        if (static_cast<unsigned>(q) < me) lo += p.sm_rate[q];
      }
      lo = warp_sum64(lo);
      all = warp_sum64(all);
      __shared__ long long red[2][NW];
      if (lane == 0) {
        red[0][warp] = lo;
        red[1][warp] = all;
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        long long a0 = 0, a1 = 0;
        for (int k = 0; k < NW; ++k) {
          a0 += red[0][k];
          a1 += red[1][k];
        }
        sm_lo = a0;
        sm_all = a1;
      }
    }
    __syncthreads();
    if (sm_ok && sm_all > 0) {
      const int smid = sm_local & 65535, local = sm_local >> 16;
      const int cps = partial ? 1 : static_cast<int>(gridDim.x) / p.num_sms;  // CTAs on every SM
      const int nsub = cps * NW, k = local * NW + warp;
      const long long lo = T * sm_lo / sm_all, hi = T * (sm_lo + p.sm_rate[smid]) / sm_all;
      ra = lo + (hi - lo) * k / nsub;
      re = lo + (hi - lo) * (k + 1) / nsub;
      r_index = smid * nsub + k;
    } else {  // an SM outside the table (cannot happen on the device that recorded it): no share
      ra = re = 0;
      r_index = gw;
      if (threadIdx.x == 0) set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
    }
  } else {
    const long long W = T < p.total_warps ? T : p.total_warps;
    if (gw < W) {
      ra = range_start(gw, T, W);
      re = range_start(gw + 1, T, W);
    }
  }
  uint64_t* bar = bars[warp];
  TileMeta* meta = metas[warp];
  uint8_t* ring = base + static_cast<size_t>(warp) * R * S::STAGE_BYTES;
  long long issued = 0, stopped_at = -1;
  int nslots = 0;

  if (ra < re) {
    if (lane == 0) {
      prefetch_tmap(&tmk);
      prefetch_tmap(&tmv);
#pragma unroll
      for (int k = 0; k < R; ++k) mbar_init(&bar[k], 1);
      fence_mbar_init();
    }
    __syncwarp();
    const uint64_t pol = policy_evict_first();

    // ---- producer: the load cursor walks the warp's range [a, e)
    const long long a = ra, e = re;
    Cursor lc;
    seek(p, pfx, a, lane, lc);
    const unsigned long long t_first = p.trace ? globaltimer_ns() : 0;
    bool loading = true;
    BtWindow win;
    win.s = -1;

    const int bs_shift = p.block_size == 32 ? 5 : 4;
    auto issue = [&](int stage) {
      const bool first = lc.u == a, last = lc.u == e - 1;
      const int key0 = lc.k0 + lc.t * TK;
      const int lb = key0 >> bs_shift, y = key0 & (p.block_size - 1);  // block_size is 16 or 32
      const int blk = bt_lookup(p, win, lc.s, lb, lane);
      // 32-key tiles: the second 16 keys come in a box of their own, when the segment has them
      bool two = false;
      int blk2 = -1, y2 = 0;
      if constexpr (TK == 2 * TILE_KEYS) {
        two = lc.t * TK + TILE_KEYS < lc.nkeys;
        if (two) {
          const int key1 = key0 + TILE_KEYS;
          y2 = key1 & (p.block_size - 1);
          blk2 = bt_lookup(p, win, lc.s, key1 >> bs_shift, lane);
        }
      }
      if (lc.t == 0 || first) {
        // warm L1 with query rows a segment ahead: the next segment's (row + 1
        // after the last KV head: rows of consecutive sequences are consecutive),
        // and at the start of a run the current one as well
        const long long row = lc.q0 + lc.i;
        const long long nq = (row + (lc.h + 1 == p.num_kv_heads)) * p.num_q_heads +
                             ((lc.h + 1) % p.num_kv_heads) * p.group;
        const long long cq = row * p.num_q_heads + lc.h * p.group;
        if (nq < static_cast<long long>(p.num_rows) * p.num_q_heads)
          for (int off = lane * 128; off < p.group * D * 2; off += 32 * 128)
            prefetch_l1(static_cast<const char*>(p.q) + nq * D * 2 + off);
        if (first)
          for (int off = lane * 128; off < p.group * D * 2; off += 32 * 128)
            prefetch_l1(static_cast<const char*>(p.q) + cq * D * 2 + off);
      }
      if (lane == 0) {
        TileMeta& m = meta[stage];
        m.u = lc.u;
        m.row = lc.q0 + lc.i;
        m.h = lc.h;
        m.t = lc.t;
        m.n = lc.n;
        m.nkeys = lc.nkeys;
        m.flags = (first ? 1 : 0) | (last ? 2 : 0);
        if (blk < 0 || blk >= p.num_blocks) set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
        if (two && (blk2 < 0 || blk2 >= p.num_blocks)) set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));
        uint8_t* st = ring + stage * S::STAGE_BYTES;
        mbar_arrive_expect_tx(&bar[stage], two ? 4 * S::BOX_BYTES : 2 * S::BOX_BYTES);
        tma_load_5d(st, &tmk, &bar[stage], 0, y, 0, lc.h, blk, pol);
        tma_load_5d(st + S::HALF_BYTES, &tmv, &bar[stage], 0, y, 0, lc.h, blk, pol);
        if (two) {  // rows 16 .. 31 of the tile (the skipped box's stale rows are masked like any past the context)
          tma_load_5d(st + S::BOX_BYTES, &tmk, &bar[stage], 0, y2, 0, lc.h, blk2, pol);
          tma_load_5d(st + S::HALF_BYTES + S::BOX_BYTES, &tmv, &bar[stage], 0, y2, 0, lc.h, blk2, pol);
        }
      }
      ++issued;
      if (!last)
        advance(p, lc);
      else
        loading = false;
    };

    for (int k = 0; k < R && loading; ++k) issue(k);
    // the first tiles are in flight: do this thread's share of the fused append meanwhile
    if (p.k_new)
      fused_append<D, F8>(p, static_cast<long long>(blockIdx.x) * ROWS_THREADS + threadIdx.x,
                      static_cast<long long>(gridDim.x) * ROWS_THREADS);

    float o[KT][NT][4];
    uint32_t qb[NT][KT][2];
    // 16-byte chunks of the newest K and V row (as the cache stores them) per lane
    constexpr int NCHUNK = F8 ? D / 16 : D / 8;
    constexpr int NEWV = (2 * NCHUNK + 31) / 32;
    uint4 newkv[NEWV];
    float m[NT][2], l[NT][2];
    bool began = false;
    int piece_t0 = 0;

    int next_stage = 0;
    uint32_t next_phase = 0;
    for (long long j = 0; j < issued; ++j) {
      const int stage = next_stage;  // j % R and (j / R) & 1, kept incrementally
      const uint32_t phase = next_phase;
      if (++next_stage == R) {
        next_stage = 0;
        next_phase ^= 1;
      }
      if (!mbar_wait(&bar[stage], phase)) {
        set_status(p.status, PA_STATUS_BIT(PA_ERR_TIMEOUT));
        stopped_at = j;
        break;
      }
      const TileMeta tm = meta[stage];
      const bool run_start = tm.flags & 1, run_end = tm.flags & 2;

      if (tm.t == 0 || run_start) {  // a piece starts: load the G query rows of this KV head
        began = (tm.t == 0);
        piece_t0 = tm.t;
        if (p.k_new) {  // fused append: the segment's newest key and value come from k_new / v_new
#pragma unroll
          for (int k = 0; k < NEWV; ++k) {
            const int ch = lane + 32 * k;
            if (ch < 2 * NCHUNK) {
              const uint4* row = reinterpret_cast<const uint4*>(ch < NCHUNK ? p.k_new : p.v_new) +
                                 (static_cast<long long>(tm.row) * p.num_kv_heads + tm.h) * (D / 8);
              if constexpr (F8) {  // 16 bf16 -> 16 codes, quantised as the append quantises them
                const float inv = ch < NCHUNK ? p.k_inv_scale : p.v_inv_scale;
                const uint2 a = quantize8(__ldg(row + 2 * (ch % NCHUNK)), inv);
                const uint2 b = quantize8(__ldg(row + 2 * (ch % NCHUNK) + 1), inv);
                newkv[k] = make_uint4(a.x, a.y, b.x, b.y);
              } else {
                newkv[k] = __ldg(row + ch % NCHUNK);
              }
            }
          }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int head = nt * 8 + g;
          const bool ok = head < p.group;
          const uint32_t* qp = reinterpret_cast<const uint32_t*>(
              static_cast<const __nv_bfloat16*>(p.q) +
              (static_cast<long long>(tm.row) * p.num_q_heads + tm.h * p.group + (ok ? head : 0)) * D);
#pragma unroll
          for (int kk = 0; kk < KT; ++kk) {
            if constexpr (F8) {
              // f16 B fragment in the head-dim order of the E4M3 K fragments:
              // k-step kk, lane column c covers head-dim 16 kk + 4c .. + 3
              const uint2 w = ok ? __ldg(reinterpret_cast<const uint2*>(qp + 8 * kk + 2 * c)) : make_uint2(0u, 0u);
              qb[nt][kk][0] = pack_f16x2(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u));
              qb[nt][kk][1] = pack_f16x2(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
            } else {
              qb[nt][kk][0] = ok ? __ldg(qp + 8 * kk + c) : 0u;
              qb[nt][kk][1] = ok ? __ldg(qp + 8 * kk + 4 + c) : 0u;
            }
          }
          m[nt][0] = m[nt][1] = -INFINITY;
          l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
          for (int mt = 0; mt < KT; ++mt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
        }
      }

      uint8_t* kt = ring + stage * S::STAGE_BYTES;
      uint8_t* vt = kt + S::HALF_BYTES;
      const int nvalid = min(TK, tm.nkeys - tm.t * TK);
      if (p.k_new && tm.t == tm.n - 1) {
        // the newest key is row nvalid - 1 of this tile: overwrite what the
        // copy brought (the append of this very launch may not have landed)
#pragma unroll
        for (int k = 0; k < NEWV; ++k) {
          const int ch = lane + 32 * k;
          if (ch < 2 * NCHUNK) {
            const int idx = ch % NCHUNK;
            *reinterpret_cast<uint4*>((ch < NCHUNK ? kt : vt) + (idx >> 3) * 2048 + sw128(nvalid - 1, idx & 7)) =
                newkv[k];
          }
        }
        __syncwarp();
      }

      if constexpr (TK == 2 * TILE_KEYS) {
        // 32-key tile (E4M3, head_dim 128, one head tile): m-tiles h = 0, 1 are
        // the tile's rows 16h .. 16h + 15, one TMA box each.  Both m-tiles'
        // codes come into registers (as in the 16-key path, K by ldmatrix and
        // V by ldmatrix.trans of byte pairs), the stage goes back to TMA, and one
        // softmax step covers the 32 keys.
        uint32_t kf2[2][KT / 2][4], vf2[2][KT / 2][4];
        const uint32_t kbase = smem_u32(kt), vbase = smem_u32(vt);
        const int rr = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int x = 0; x < KT; x += 2) {
            const int ch = x + (lane >> 4);
            ldsm_x4(kbase + h * S::BOX_BYTES + sw128(rr, ch), kf2[h][x / 2][0], kf2[h][x / 2][1], kf2[h][x / 2][2],
                    kf2[h][x / 2][3]);
            ldsm_x4_trans(vbase + h * S::BOX_BYTES + sw128(rr, ch), vf2[h][x / 2][0], vf2[h][x / 2][1],
                          vf2[h][x / 2][2], vf2[h][x / 2][3]);
          }
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // V rows of keys past the context: exact zeros (P = 0 times NaN is NaN)
          const int nv = nvalid - TILE_KEYS * h;
          if (nv < TILE_KEYS) {
            const uint32_t lo = (2 * c < nv ? 0x0000ffffu : 0u) | (2 * c + 1 < nv ? 0xffff0000u : 0u);
            const uint32_t hi = (2 * c + 8 < nv ? 0x0000ffffu : 0u) | (2 * c + 9 < nv ? 0xffff0000u : 0u);
#pragma unroll
            for (int x = 0; x < KT / 2; ++x) {
              vf2[h][x][0] &= lo;
              vf2[h][x][1] &= hi;
              vf2[h][x][2] &= lo;
              vf2[h][x][3] &= hi;
            }
          }
        }
        __syncwarp();
        if (loading) {
          if (lane == 0) fence_proxy_async_smem();
          issue(stage);
        }

        // S^T[key, head] = K . Q^T for each m-tile
        float sv[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int x = 0; x < KT / 2; ++x) {
            const uint32_t* r = kf2[h][x];
            const uint32_t a0 = e4m3x2_lo_to_f16x2(r[0]), a1 = e4m3x2_lo_to_f16x2(r[1]);
            const uint32_t a2 = e4m3x2_hi_to_f16x2(r[0]), a3 = e4m3x2_hi_to_f16x2(r[1]);
            const uint32_t b0 = e4m3x2_lo_to_f16x2(r[2]), b1 = e4m3x2_lo_to_f16x2(r[3]);
            const uint32_t b2 = e4m3x2_hi_to_f16x2(r[2]), b3 = e4m3x2_hi_to_f16x2(r[3]);
            mma_f16_16816(acc, a0, a1, a2, a3, qb[0][2 * x][0], qb[0][2 * x][1]);
            mma_f16_16816(acc, b0, b1, b2, b3, qb[0][2 * x + 1][0], qb[0][2 * x + 1][1]);
          }
          // this lane: keys 16h + g and 16h + g + 8 of heads 2c, 2c + 1
          sv[h][0] = acc[0] * p.scale_log2;
          sv[h][1] = acc[1] * p.scale_log2;
          sv[h][2] = acc[2] * p.scale_log2;
          sv[h][3] = acc[3] * p.scale_log2;
          if (TILE_KEYS * h + g >= nvalid) sv[h][0] = sv[h][1] = -INFINITY;
          if (TILE_KEYS * h + g + 8 >= nvalid) sv[h][2] = sv[h][3] = -INFINITY;
        }

        // online softmax over the 32 keys
        float mx0 = fmaxf(fmaxf(sv[0][0], sv[0][2]), fmaxf(sv[1][0], sv[1][2]));
        float mx1 = fmaxf(fmaxf(sv[0][1], sv[0][3]), fmaxf(sv[1][1], sv[1][3]));
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(FULL_MASK, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(FULL_MASK, mx1, off));
        }
        const float mn0 = fmaxf(m[0][0], mx0), mn1 = fmaxf(m[0][1], mx1);
        const bool moved = (mn0 != m[0][0]) | (mn1 != m[0][1]);
        const float al0 = fast_exp2(m[0][0] - mn0), al1 = fast_exp2(m[0][1] - mn1);
        m[0][0] = mn0;
        m[0][1] = mn1;
        uint32_t pb2[2][2];
        float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float p0 = fast_exp2(sv[h][0] - mn0), p2 = fast_exp2(sv[h][2] - mn0);
          const float p1 = fast_exp2(sv[h][1] - mn1), p3 = fast_exp2(sv[h][3] - mn1);
          ls0 += p0 + p2;
          ls1 += p1 + p3;
          pb2[h][0] = movmatrix_trans(pack_f16x2(p0, p1));  // P in f16 for the f16 MMA
          pb2[h][1] = movmatrix_trans(pack_f16x2(p2, p3));
        }
        l[0][0] = l[0][0] * al0 + ls0;
        l[0][1] = l[0][1] * al1 + ls1;
        if (__any_sync(FULL_MASK, moved)) {  // rescale O only when some running maximum grew
#pragma unroll
          for (int mt = 0; mt < KT; ++mt) {
            o[mt][0][0] *= al0;
            o[mt][0][1] *= al1;
            o[mt][0][2] *= al0;
            o[mt][0][3] *= al1;
          }
        }

        // O^T[d, head] += V^T . P^T, one k-step of 16 keys per m-tile
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int x = 0; x < KT / 2; ++x) {
            const uint32_t r0 = pair_bytes(vf2[h][x][0]), r1 = pair_bytes(vf2[h][x][1]);
            const uint32_t r2 = pair_bytes(vf2[h][x][2]), r3 = pair_bytes(vf2[h][x][3]);
            const uint32_t a0 = e4m3x2_lo_to_f16x2(r0), a1 = e4m3x2_hi_to_f16x2(r0);
            const uint32_t a2 = e4m3x2_lo_to_f16x2(r1), a3 = e4m3x2_hi_to_f16x2(r1);
            const uint32_t b0 = e4m3x2_lo_to_f16x2(r2), b1 = e4m3x2_hi_to_f16x2(r2);
            const uint32_t b2 = e4m3x2_lo_to_f16x2(r3), b3 = e4m3x2_hi_to_f16x2(r3);
            mma_f16_16816(o[2 * x][0], a0, a1, a2, a3, pb2[h][0], pb2[h][1]);
            mma_f16_16816(o[2 * x + 1][0], b0, b1, b2, b3, pb2[h][0], pb2[h][1]);
          }
      } else {
        // Pull the tile into registers (K as the A operand of S^T = K Q^T, V^T via
        // ldmatrix.trans as the A operand of O^T += V^T P^T) and hand the stage
        // back to TMA at once, so the ring never waits on the math.  With
        // head_dim 256 both bf16 fragments would not fit in registers: V is read
        // after the softmax and the stage is released then (E4M3 codes, one byte
        // each, fit).
        constexpr bool kEarly = D <= 128 || F8;
        uint32_t kf[KT][4], vf[KT][4];
        const int mi = lane >> 3;
        const uint32_t kbase = smem_u32(kt), vbase = smem_u32(vt);
        auto load_v = [&]() {
          if constexpr (F8) {
            // E4M3 V: one ldmatrix.trans of byte pairs covers m-tiles X, X + 1
            // (16-byte chunks X, X + 1 = head-dim 16X .. 16X + 31) for keys 0-7
            // and 8-15.  A lane receives keys 2c, 2c+1 at head-dim 2g, 2g+1 of
            // the chunk.  The bytes stay packed in vf[X / 2]; the product loop
            // pairs them by head-dim into the f16 A rows g (head-dim 16X + 2g)
            // and g + 8 (head-dim 16X + 2g + 1).
            const int rv = (lane & 7) + ((lane >> 3) & 1) * 8;
  #pragma unroll
            for (int x = 0; x < KT; x += 2) {
              const int ch = x + (lane >> 4);
              ldsm_x4_trans(vbase + (ch >> 3) * 2048 + sw128(rv, ch & 7), vf[x / 2][0], vf[x / 2][1], vf[x / 2][2],
                            vf[x / 2][3]);
            }
          } else {
            const int rv = (lane & 7) + (mi >> 1) * 8;
  #pragma unroll
            for (int mt = 0; mt < KT; ++mt) {
              const int cg = 2 * mt + (mi & 1);
              ldsm_x4_trans(vbase + (cg >> 3) * 2048 + sw128(rv, cg & 7), vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3]);
            }
          }
          if (nvalid < TILE_KEYS) {
            // keys past the context may hold anything (even NaN): their V rows must
            // be exact zeros, since P = 0 times NaN is NaN.  This lane holds keys
            // 2c, 2c+1 (fragments 0, 1) and 8+2c, 9+2c (fragments 2, 3).
            const uint32_t lo = (2 * c < nvalid ? 0x0000ffffu : 0u) | (2 * c + 1 < nvalid ? 0xffff0000u : 0u);
            const uint32_t hi = (2 * c + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * c + 9 < nvalid ? 0xffff0000u : 0u);
            if constexpr (F8) {  // packed codes: registers 0, 2 hold keys 2c, 2c+1 and 1, 3 keys 8+2c, 9+2c
  #pragma unroll
              for (int x = 0; x < KT / 2; ++x) {
                vf[x][0] &= lo;
                vf[x][1] &= hi;
                vf[x][2] &= lo;
                vf[x][3] &= hi;
              }
            } else {
  #pragma unroll
              for (int mt = 0; mt < KT; ++mt) {
                vf[mt][0] &= lo;
                vf[mt][1] &= lo;
                vf[mt][2] &= hi;
                vf[mt][3] &= hi;
              }
            }
          }
        };
        auto release = [&]() {
          __syncwarp();
          if (loading) {
            if (lane == 0) fence_proxy_async_smem();
            issue(stage);
          }
        };
        if constexpr (F8) {
          // E4M3 K: one ldmatrix of byte pairs covers k-steps X, X + 1 (16-byte
          // chunks X, X + 1) for keys 0-7 and 8-15.  A lane receives head-dim
          // 4c .. 4c+3 of the chunk; its low pair is the f16 A column pair 2c, 2c+1
          // of the k-step and its high pair the pair 2c+8, 2c+9 (Q uses the same
          // order).  The codes stay packed in kf[X / 2] until the product loop.
          const int rk = (lane & 7) + ((lane >> 3) & 1) * 8;
  #pragma unroll
          for (int x = 0; x < KT; x += 2) {
            const int ch = x + (lane >> 4);
            ldsm_x4(kbase + (ch >> 3) * 2048 + sw128(rk, ch & 7), kf[x / 2][0], kf[x / 2][1], kf[x / 2][2],
                    kf[x / 2][3]);
          }
        } else {
          const int rk = (lane & 7) + (mi & 1) * 8;
  #pragma unroll
          for (int kk = 0; kk < KT; ++kk)
            ldsm_x4(kbase + (kk >> 2) * 2048 + sw128(rk, 2 * (kk & 3) + (mi >> 1)), kf[kk][0], kf[kk][1], kf[kk][2],
                    kf[kk][3]);
        }
        if constexpr (kEarly) {
          load_v();
          release();
        }

        // S^T[key, head] = K . Q^T
        float sacc[NT][4];
  #pragma unroll
        for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
        if constexpr (F8) {  // E4M3 -> f16 just before each pair of k-steps
  #pragma unroll
          for (int x = 0; x < KT / 2; ++x) {
            const uint32_t* r = kf[x];
            const uint32_t a0 = e4m3x2_lo_to_f16x2(r[0]), a1 = e4m3x2_lo_to_f16x2(r[1]);
            const uint32_t a2 = e4m3x2_hi_to_f16x2(r[0]), a3 = e4m3x2_hi_to_f16x2(r[1]);
            const uint32_t b0 = e4m3x2_lo_to_f16x2(r[2]), b1 = e4m3x2_lo_to_f16x2(r[3]);
            const uint32_t b2 = e4m3x2_hi_to_f16x2(r[2]), b3 = e4m3x2_hi_to_f16x2(r[3]);
  #pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mma_f16_16816(sacc[nt], a0, a1, a2, a3, qb[nt][2 * x][0], qb[nt][2 * x][1]);
              mma_f16_16816(sacc[nt], b0, b1, b2, b3, qb[nt][2 * x + 1][0], qb[nt][2 * x + 1][1]);
            }
          }
        } else if constexpr (ROWS_S_CHAINS == 2) {
          // two independent accumulation chains (even and odd k-steps), summed:
          // half the dependent MMA latency on the per-tile critical path
          float sacc2[NT][4];
  #pragma unroll
          for (int nt = 0; nt < NT; ++nt) sacc2[nt][0] = sacc2[nt][1] = sacc2[nt][2] = sacc2[nt][3] = 0.f;
  #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
            for (int kk = 0; kk < KT; kk += 2) {
              mma_bf16_16816(sacc[nt], kf[kk][0], kf[kk][1], kf[kk][2], kf[kk][3], qb[nt][kk][0], qb[nt][kk][1]);
              mma_bf16_16816(sacc2[nt], kf[kk + 1][0], kf[kk + 1][1], kf[kk + 1][2], kf[kk + 1][3], qb[nt][kk + 1][0],
                             qb[nt][kk + 1][1]);
            }
  #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
            for (int r = 0; r < 4; ++r) sacc[nt][r] += sacc2[nt][r];
        } else {
  #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
            for (int kk = 0; kk < KT; ++kk)
              mma_bf16_16816(sacc[nt], kf[kk][0], kf[kk][1], kf[kk][2], kf[kk][3], qb[nt][kk][0], qb[nt][kk][1]);
        }

        // online softmax on the fragment: this lane holds keys g, g+8 of heads 2c, 2c+1
        uint32_t pb[NT][2];
        float al[NT][2];
        bool moved = false;
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
          moved |= (mn0 != m[nt][0]) | (mn1 != m[nt][1]);
          al[nt][0] = fast_exp2(m[nt][0] - mn0);
          al[nt][1] = fast_exp2(m[nt][1] - mn1);
          m[nt][0] = mn0;
          m[nt][1] = mn1;
          const float p0 = fast_exp2(s0 - mn0), p2 = fast_exp2(s2 - mn0);
          const float p1 = fast_exp2(s1 - mn1), p3 = fast_exp2(s3 - mn1);
          l[nt][0] = l[nt][0] * al[nt][0] + p0 + p2;
          l[nt][1] = l[nt][1] * al[nt][1] + p1 + p3;
          if constexpr (F8) {  // P in f16 for the f16 MMA
            pb[nt][0] = movmatrix_trans(pack_f16x2(p0, p1));
            pb[nt][1] = movmatrix_trans(pack_f16x2(p2, p3));
          } else {
            pb[nt][0] = movmatrix_trans(pack_bf16x2(p0, p1));
            pb[nt][1] = movmatrix_trans(pack_bf16x2(p2, p3));
          }
        }
        if (__any_sync(FULL_MASK, moved)) {  // rescale O only when some running maximum grew
  #pragma unroll
          for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
            for (int mt = 0; mt < KT; ++mt) {
              o[mt][nt][0] *= al[nt][0];
              o[mt][nt][1] *= al[nt][1];
              o[mt][nt][2] *= al[nt][0];
              o[mt][nt][3] *= al[nt][1];
            }
        }

        // O^T[d, head] += V^T . P^T
        if constexpr (!kEarly) {
          load_v();
          release();
        }
        if constexpr (F8) {  // pair the codes by head-dim, E4M3 -> f16, two m-tiles per packed fragment
  #pragma unroll
          for (int x = 0; x < KT / 2; ++x) {
            const uint32_t r0 = pair_bytes(vf[x][0]), r1 = pair_bytes(vf[x][1]);
            const uint32_t r2 = pair_bytes(vf[x][2]), r3 = pair_bytes(vf[x][3]);
            const uint32_t a0 = e4m3x2_lo_to_f16x2(r0), a1 = e4m3x2_hi_to_f16x2(r0);
            const uint32_t a2 = e4m3x2_lo_to_f16x2(r1), a3 = e4m3x2_hi_to_f16x2(r1);
            const uint32_t b0 = e4m3x2_lo_to_f16x2(r2), b1 = e4m3x2_hi_to_f16x2(r2);
            const uint32_t b2 = e4m3x2_lo_to_f16x2(r3), b3 = e4m3x2_hi_to_f16x2(r3);
  #pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mma_f16_16816(o[2 * x][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
              mma_f16_16816(o[2 * x + 1][nt], b0, b1, b2, b3, pb[nt][0], pb[nt][1]);
            }
          }
        } else {
  #pragma unroll
          for (int mt = 0; mt < KT; ++mt)
  #pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma_bf16_16816(o[mt][nt], vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3], pb[nt][0], pb[nt][1]);
        }
      }

      // ---- end of a piece: write the output, or a partial linked to its segment
      if (tm.t == tm.n - 1 || run_end) {
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
        if (began && tm.t == tm.n - 1 && p.num_groups > 0 && seq_info(p, tm.row).k0 > 0) {
          // the whole private part of a shared-prefix segment: keep it unnormalised
          // for the merge phase, which folds in the prefix (decode: row = sequence)
          store_own_partial<D, NT>(p, o, m, l, tm.row, tm.h, lane);
          if (lane == 0)
            p.seginfo[static_cast<long long>(tm.row) * p.num_kv_heads + tm.h] = (tm.u - tm.t) + 1;  // no pieces
        } else if (began && tm.t == tm.n - 1) {
          store_output<D, NT, F8>(p, o, l, tm.row, tm.h, lane);
        } else if (nslots < ROWS_SLOTS_PER_WARP) {
          const long long slot = static_cast<long long>(r_index) * ROWS_SLOTS_PER_WARP + nslots++;
          float* ps = p.partials + slot * S::SLOT_FLOATS;
#pragma unroll
          for (int mt = 0; mt < KT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              reinterpret_cast<float4*>(ps)[(mt * NT + nt) * 32 + lane] =
                  make_float4(o[mt][nt][0], o[mt][nt][1], o[mt][nt][2], o[mt][nt][3]);
          if (lane < 4) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              ps[S::SLOT_M + nt * 8 + 2 * lane] = m[nt][0];
              ps[S::SLOT_M + nt * 8 + 2 * lane + 1] = m[nt][1];
              ps[S::SLOT_L + nt * 8 + 2 * lane] = l[nt][0];
              ps[S::SLOT_L + nt * 8 + 2 * lane + 1] = l[nt][1];
            }
          }
          // record the piece at its first unit and mark its segment; the
          // segment is merged after the grid barrier (plain stores, no waiting)
          if (lane == 0) {
            const long long segA = tm.u - tm.t;
            p.table[segA + piece_t0] = (static_cast<long long>(tm.t - piece_t0 + 1) << 32) | slot;
            p.seginfo[static_cast<long long>(tm.row) * p.num_kv_heads + tm.h] =
                (static_cast<long long>(tm.n) << 40) | (segA + 1);
          }
        } else {
          set_status(p.status, PA_STATUS_BIT(PA_ERR_RANGE));  // cannot happen: slots cover every run end
        }
      }
    }

    if (p.trace && lane == 0) {  // calibration: when this warp's range streamed, and on which SM
      unsigned smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      unsigned long long* tr = p.trace + static_cast<long long>(r_index) * 4;
      tr[0] = smid;
      tr[1] = static_cast<unsigned long long>(e - a);
      tr[2] = t_first;
      tr[3] = globaltimer_ns();
    }
    if (stopped_at >= 0) {  // let copies still in flight land before the shared memory goes away
      for (long long j = stopped_at + 1; j < issued; ++j) mbar_wait(&bar[j % R], static_cast<uint32_t>((j / R) & 1));
    }
  }

  if (!(ra < re) && p.k_new)  // warps without tiles still take their share of the fused append
    fused_append<D, F8>(p, static_cast<long long>(blockIdx.x) * ROWS_THREADS + threadIdx.x,
                    static_cast<long long>(gridDim.x) * ROWS_THREADS);
  if (T == 0) {  // no tile anywhere (every CTA sees the same T): nothing to merge, no barrier
    if (p.weighted && threadIdx.x == 0 && sm_id < static_cast<unsigned>(p.num_sms)) {  // undo the registration
      if (partial) {
        atomicAnd(p.sm_mask + (sm_id >> 5), ~(1u << (sm_id & 31)));
        atomicSub(p.sched + 2, 1);
      } else {
        atomicSub(p.sm_slots + sm_id, 1);
      }
    }
    return;
  }

  // ---- grid barrier: every partial and table entry is stored before any merge reads it
  __syncwarp();
  if (lane == 0) {
    __threadfence();
    atomicAdd(p.sched, 1);
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(p.sched) < p.total_warps) {
      if (globaltimer_ns() - t0 > WAIT_NS) {
        set_status(p.status, PA_STATUS_BIT(PA_ERR_TIMEOUT));
        break;
      }
      __nanosleep(64);
    }
  }
  __syncwarp();

  // ---- merge every segment that has partial pieces
  const long long nseg = static_cast<long long>(p.num_rows) * p.num_kv_heads;
  for (long long seg = gw; seg < nseg; seg += p.total_warps) {
    const long long info = __ldcg(p.seginfo + seg);
    if (info == 0) continue;
    merge_segment<D, NT, F8>(p, (info & ((1ll << 40) - 1)) - 1, static_cast<int>(info >> 40),
                         static_cast<int>(seg / p.num_kv_heads), static_cast<int>(seg % p.num_kv_heads), lane);
    if (lane == 0) p.seginfo[seg] = 0;
  }

  // ---- the last warp out puts the barrier words back to zero
  __syncwarp();
  if (lane == 0) {
    const int out = atomicAdd(p.sched + 1, 1);
    if (out == p.total_warps - 1) {
      p.sched[0] = 0;
      p.sched[1] = 0;
      if (p.weighted) {
        p.sched[2] = 0;
        for (int q = 0; q < 8; ++q) p.sm_mask[q] = 0;
        for (int q = 0; q < p.num_sms; ++q) p.sm_slots[q] = 0;
      }
    }
  }
}

// ------------------------------------------------------------------ host side

template <int D, int NT, int R, bool F8 = false, int TK = TILE_KEYS, int NW = ROWS_WARPS>
static int launch_rows_t(const RowsParams& p0, const CUtensorMap& tmk, const CUtensorMap& tmv, cudaStream_t stream,
                         int num_sms, int ctas) {
  constexpr int ROWS_THREADS = NW * 32;
  using S = RowsShape<D, NT, F8, TK>;
  const int smem = NW * R * S::STAGE_BYTES + 1024 + (ROWS_SMEM_SEQS + 1) * 8;
  auto kern = rows_kernel<D, NT, R, F8, TK, NW>;
  static PerDevice configured;  // CTAs per SM on each device
  int blocks_per_sm = 0;
  const int rc_setup = per_device(
      configured,
      [&](int) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, ROWS_THREADS, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
        if (nb < 1) return static_cast<int>(PA_ERR_CUDA);
        constexpr int cap = rows_ctas_per_sm<D, NT, F8, TK>();
        return nb > cap ? cap : nb;
      },
      &blocks_per_sm);
  if (rc_setup != PA_OK) return rc_setup;
  RowsParams p = p0;
  p.tile_shift = TK == 32 ? 5 : 4;
  // The per-SM weights hold for the variant they were measured with (bf16,
  // head_dim 128, one head tile, two 4-warp CTAs per SM over the whole GPU):
  // on the other variants they made steps slower (head_dim 256 by 10 %, the
  // E4M3 kernel by 4 %), so those split equally.
  if (!(D == 128 && NT == 1 && !F8 && NW == ROWS_WARPS && ctas <= 0)) p.weighted = 0;
  // ctas > 0: a launch on part of the GPU (one CTA per SM, the rest of the
  // SMs left to a kernel that runs beside it)
  const int grid = ctas > 0 ? (ctas < num_sms * blocks_per_sm ? ctas : num_sms * blocks_per_sm)
                            : num_sms * blocks_per_sm;
  p.total_warps = grid * NW;
  // Programmatic dependent launch: the prologue (a scan of the batch
  // metadata) overlaps the kernel before it, typically the cache append;
  // the kernel waits for that grid before it reads the cache.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(ROWS_THREADS);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  // Cooperative: every CTA is resident at once, which the grid barrier before
  // the merge phase relies on.
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return check_launch(cudaLaunchKernelEx(&cfg, kern, tmk, tmv, p), "rows_kernel launch");
}

int rows_supported(int group, int head_dim) {
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return 0;
  if (group < 1) return 0;
  if (head_dim == 256) return group <= 8;
  return group <= 16;
}

namespace {
size_t round256(size_t n) { return (n + 255) / 256 * 256; }
// [0] warps at the barrier, [1] warps done, [2] CTAs of a partial launch that
// have registered their SM, [8..15] their SM mask, [16..16 + 256) CTAs per SM
// that have taken their share
constexpr size_t SCHED_BYTES = 2048;
size_t slot_bytes(int group, int head_dim) {
  const int nt = group > 8 ? 2 : 1;
  const size_t o = static_cast<size_t>(head_dim / 16) * nt * 32 * 4;
  return (o + 16 * nt + 1 + 63) / 64 * 64 * sizeof(float);
}
size_t max_warps(int num_sms) { return static_cast<size_t>(num_sms) * ROWS_MAX_CTAS_PER_SM * ROWS_WARPS; }
static_assert(ROWS_WARPS_WIDE <= ROWS_MAX_CTAS_PER_SM * ROWS_WARPS, "partial slots per SM");
}  // namespace

namespace {
size_t table_entries(int num_rows, int num_kv_heads, long long max_keys) {
  return static_cast<size_t>(num_rows) * num_kv_heads * static_cast<size_t>((max_keys + TILE_KEYS - 1) / TILE_KEYS);
}
}  // namespace

// Partial-result area: the rows kernel's slots, which the multi-row kernel
// (head_dim 128) also uses for its pieces (it runs to completion first).
static size_t partials_bytes(int num_q_heads, int num_kv_heads, int head_dim, int num_sms) {
  const size_t rows = max_warps(num_sms) * ROWS_SLOTS_PER_WARP * slot_bytes(num_q_heads / num_kv_heads, head_dim);
  const size_t verify = static_cast<size_t>(num_sms) * 2 * verify_slot_floats(VERIFY_MAX_COLS) * sizeof(float);
  return head_dim == 128 && verify > rows ? verify : rows;
}

static size_t verify_counter_bytes(int num_sms) { return round256(static_cast<size_t>(num_sms) * sizeof(int)); }

size_t rows_workspace_bytes(int num_rows, int num_q_heads, int num_kv_heads, int head_dim, long long max_keys,
                            int num_sms) {
  return SCHED_BYTES + verify_counter_bytes(num_sms) +
         round256(static_cast<size_t>(num_rows) * num_kv_heads * sizeof(long long)) +
         round256(table_entries(num_rows, num_kv_heads, max_keys) * sizeof(long long)) +
         partials_bytes(num_q_heads, num_kv_heads, head_dim, num_sms);
}

void rows_workspace_layout(void* ws, int num_rows, int num_q_heads, int num_kv_heads, int head_dim,
                           long long max_keys, int num_sms, RowsParams* p) {
  (void)num_q_heads;
  (void)head_dim;
  uint8_t* b = static_cast<uint8_t*>(ws);
  p->sched = reinterpret_cast<int*>(b);
  p->sm_mask = reinterpret_cast<unsigned*>(b) + 8;
  p->sm_slots = reinterpret_cast<int*>(b) + 16;
  b += SCHED_BYTES;
  p->verify_counters = reinterpret_cast<int*>(b);
  b += verify_counter_bytes(num_sms);
  p->seginfo = reinterpret_cast<long long*>(b);
  b += round256(static_cast<size_t>(num_rows) * num_kv_heads * sizeof(long long));
  p->table = reinterpret_cast<long long*>(b);
  p->table_len = static_cast<long long>(table_entries(num_rows, num_kv_heads, max_keys));
  b += round256(table_entries(num_rows, num_kv_heads, max_keys) * sizeof(long long));
  p->partials = reinterpret_cast<float*>(b);
  p->num_rows = num_rows;
}

int launch_rows(const RowsParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, int head_dim,
                cudaStream_t stream, int num_sms, int ctas) {
  const bool two = p.group > 8;
  if (p.kv_fp8) {  // E4M3 caches: a tile is half the bytes, so more stages (or more CTAs) per SM
    switch (head_dim) {
      case 128:
        return two ? launch_rows_t<128, 2, 6, true>(p, tmk, tmv, stream, num_sms, 0)
                   : launch_rows_t<128, 1, 3, true, 32>(p, tmk, tmv, stream, num_sms, 0);
      case 256:
        return launch_rows_t<256, 1, 3, true>(p, tmk, tmv, stream, num_sms, 0);
      default:
        return PA_ERR_UNSUPPORTED;
    }
  }
  if (ctas > 0) {  // part of the GPU, one 8-warp CTA per SM (head_dim 128: the tcgen05 chunk path's shapes)
    if (head_dim != 128) return PA_ERR_UNSUPPORTED;
    return two ? launch_rows_t<128, 2, 3, false, TILE_KEYS, ROWS_WARPS_WIDE>(p, tmk, tmv, stream, num_sms, ctas)
               : launch_rows_t<128, 1, 3, false, TILE_KEYS, ROWS_WARPS_WIDE>(p, tmk, tmv, stream, num_sms, ctas);
  }
  switch (head_dim) {
    case 64:
      return two ? launch_rows_t<64, 2, 8>(p, tmk, tmv, stream, num_sms, 0)
                 : launch_rows_t<64, 1, 8>(p, tmk, tmv, stream, num_sms, 0);
    case 128:
      return two ? launch_rows_t<128, 2, 3>(p, tmk, tmv, stream, num_sms, 0)
                 : launch_rows_t<128, 1, 3>(p, tmk, tmv, stream, num_sms, 0);
    case 256:
      return launch_rows_t<256, 1, 3>(p, tmk, tmv, stream, num_sms, 0);
    default:
      return PA_ERR_UNSUPPORTED;
  }
}

}  // namespace pa
