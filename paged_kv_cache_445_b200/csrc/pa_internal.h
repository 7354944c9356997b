// pa_internal.h -- host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "pa.h"

namespace pa {

// A CUDA call failed: remember its error for pa_last_cuda_error() (per host
// thread) and return PA_ERR_CUDA.
int cuda_fail(cudaError_t e, const char* call);
int cu_fail(CUresult r, const char* call);
// The result of a kernel launch: the launch call's own error, else the
// thread's last runtime error (a launch-configuration error, or a sticky error
// left by an earlier kernel that faulted).
inline int check_launch(cudaError_t launch_rc, const char* what) {
  if (launch_rc != cudaSuccess) {
    (void)cudaGetLastError();
    return cuda_fail(launch_rc, what);
  }
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : cuda_fail(e, what);
}

// Per-device launch set-up of one kernel (its shared-memory opt-in, its CTAs
// per SM), done once per device and safe under concurrent callers: the value
// is an atomic, and two threads that set the same device up at once both make
// the same idempotent CUDA calls and store the same value.
constexpr int PA_MAX_DEVICES = 64;
struct PerDevice {
  std::atomic<int> value[PA_MAX_DEVICES];  // 0: not set up on that device yet
};

// The current device's value of `cache`, computed by setup() (a positive
// value, else a pa_status) the first time.  Returns a pa_status.
template <class Setup>
int per_device(PerDevice& cache, Setup setup, int* out) {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= PA_MAX_DEVICES) return PA_ERR_CUDA;
  int v = cache.value[dev].load(std::memory_order_acquire);
  if (v <= 0) {
    v = setup(dev);
    if (v <= 0) return v < 0 ? v : PA_ERR_CUDA;
    cache.value[dev].store(v, std::memory_order_release);
  }
  *out = v;
  return PA_OK;
}

// SMs whose rates a decode launch can carry in its parameters.
constexpr int PA_MAX_WEIGHTED_SMS = 160;

// The per-SM rates pa_calibrate recorded for the current device (false if
// none, or recorded for another SM count).
bool sm_rates_snapshot(uint16_t* out, int num_sms);
void sm_rates_clear();

// Batch size up to which the rows kernel keeps per-sequence prefix sums of
// tile counts in shared memory (larger batches scan context_lens instead).
constexpr int ROWS_SMEM_SEQS_HOST = 1024;

// Parameters of the single-row attention kernel (decode rows, and the rows of
// any sequence the chunk kernel does not take).
struct RowsParams {
  void* out;                    // bf16 [Tq, Hq, D]
  const void* q;                // bf16 [Tq, Hq, D]
  const int32_t* block_tables;  // [B, max_blocks]
  const int32_t* context_lens;  // [B]
  const int32_t* query_start;   // [B + 1], or nullptr: one query row per sequence
  int num_seqs;
  int max_blocks;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int block_size;
  int num_blocks;
  int skip_multi;   // 1: sequences with more than one query row belong to the chunk kernel
  float scale_log2; // softmax scale * log2(e)
  float* partials;             // workspace: partial-result slots, two per warp
  long long* seginfo;          // workspace: (tiles << 40 | first unit + 1) of segments with partials, zero between calls
  long long* table;            // workspace: (tiles << 32 | slot) of the piece that starts at each unit
  long long table_len;         // entries in table
  int* sched;                  // workspace: [warps at the barrier, warps done], zero between calls
  int* verify_counters;        // workspace: one per SM for the multi-row kernel, zero between calls
  int num_rows;                // query rows (Tq)
  int* status;      // optional device status word
  int total_warps;
  int tile_shift;   // log2 of the keys per work unit (16, or 32 for the E4M3 kernel with one head tile)
  int trigger_early;  // 1: release the dependent grid (the chunk kernel beside this one) once the append is visible
  // Split of the tiles by SM rate (pa_calibrate): each SM takes a share in
  // proportion to sm_rate[smid], cut equally between its warps.
  int weighted;
  int num_sms;
  int* sm_slots;          // workspace: CTAs that have taken their SM's share, per SM; zero between calls
  unsigned* sm_mask;      // workspace: SMs of a launch on part of the GPU (8 words); zero between calls
  uint16_t sm_rate[PA_MAX_WEIGHTED_SMS];
  uint32_t sm_prefix[PA_MAX_WEIGHTED_SMS + 1];  // sm_prefix[s] = sum of sm_rate[0 .. s-1] (a whole-GPU launch)
  // Calibration only (nullptr otherwise): per range r, {SM id, units, time of
  // the first copy, time the last tile was consumed} (globaltimer ns).
  unsigned long long* trace;
  // Fused cache append (decode only; nullptr: none).  Row s of k_new / v_new
  // ([B, Hkv, D] bf16) is sequence s's newest token: the kernel writes it to
  // position context_lens[s] - 1 through the block table and attends to it
  // from these rows, not from the cache.
  const void* k_new;
  const void* v_new;
  void* k_cache;
  void* v_cache;
  // Shared-prefix groups (decode only; num_groups = 0: none).  Sequences
  // group_start[g] .. group_start[g+1]-1 share their first group_prefix[g]
  // tokens; the cascade kernel has attended to the first cascade_span() of
  // them and left per-slice partials in casc_partials, which this kernel folds
  // in.  Its own segments start at that key.
  const int32_t* group_start;
  const int32_t* group_prefix;
  int num_groups;
  // FP8 (E4M3) cache: codes of value / scale.  The K scale is folded into
  // scale_log2; v_scale multiplies the output; the inverse scales quantise the
  // fused append.
  int kv_fp8;
  float v_scale;
  float k_inv_scale;
  float v_inv_scale;
  const float* casc_partials;  // [B][Hq][CASCADE_SPLITS + 1][D + 4]: O, m (log2 units), l; the last slot
                               // holds this kernel's own unnormalised result of an unsplit segment
};

// Shared-prefix pass: prefix keys handled together, in tiles of 64, cut into at
// most CASCADE_SPLITS slices per group.
constexpr int CASCADE_SPLITS = 8;
constexpr int CASCADE_TILE = 64;
// one partial record: O[D], m, l, two floats of padding (16-byte aligned records)
__host__ __device__ constexpr int cascade_record_floats(int head_dim) { return head_dim + 4; }
__host__ __device__ __forceinline__ int cascade_span(int prefix_tokens) {
  return prefix_tokens >= CASCADE_TILE ? prefix_tokens / CASCADE_TILE * CASCADE_TILE : 0;
}
__host__ __device__ __forceinline__ int cascade_splits(int span) {
  const int tiles = span / CASCADE_TILE;
  if (tiles <= 0) return 0;
  const int n = tiles < CASCADE_SPLITS ? tiles : CASCADE_SPLITS;
  const int per = (tiles + n - 1) / n;
  return (tiles + per - 1) / per;  // no empty slice
}

// Sequences per M-tile of the shared-prefix pass: as many as fit in 128 rows
// with a row count that is a multiple of 8 (whole 8-row swizzle atoms: a TMA
// box of another height left the last rows of Q landing after the barrier).
__host__ __device__ __forceinline__ int cascade_tokm(int group) {
  int t = 128 / group;
  while (t > 1 && (t * group) % 8 != 0) --t;
  return t;
}

struct CascadeParams {
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* group_start;
  const int32_t* group_prefix;
  int num_groups;
  int num_q_heads;
  int num_kv_heads;
  int group;  // query heads per KV head
  int block_size;
  int num_blocks;
  float scale_log2;
  float* partials;
  int* status;
};

// Parameters of the tcgen05 chunk kernel (sequences with more than one query row).
// Sequences with 2 .. 64/G query rows (multi-token verification) on the
// tcgen05 kernel with the keys in M; the rest of a varlen batch goes to the
// chunk and rows kernels.  head_dim 128, bf16 caches.
constexpr int VERIFY_SMEM_SEQS = 512;   // batches up to this many sequences
__host__ __device__ constexpr int verify_slot_floats(int ncol) { return (ncol * 128 + 2 * ncol + 63) / 64 * 64; }
constexpr int VERIFY_MAX_COLS = 64;

struct VerifyParams {
  void* out;                    // bf16 [Tq, Hq, 128]
  const int32_t* block_tables;  // [B, max_blocks]
  const int32_t* context_lens;  // [B]
  const int32_t* query_start;   // [B + 1]
  int num_seqs;
  int max_blocks;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int block_size;
  int num_blocks;
  float scale_log2;
  int* status;
  float* slots;     // workspace: two (O, m, l) piece slots per CTA
  int* counters;    // workspace: one per CTA, zero between calls
  int ncol_lo, ncol_hi;  // set per launch: this kernel takes qlen * G in (ncol_lo, ncol_hi]
};

int verify_supported(int group, int head_dim, int num_seqs);
// which: bit 0 launches the 32-column kernel, bit 1 the 64-column one.
int launch_verify(const VerifyParams& p, const void* q, const void* k_cache, const void* v_cache,
                  int total_q_tokens, cudaStream_t stream, int num_sms, int which = 3);

struct ChunkParams {
  void* out;                    // bf16 [Tq, Hq, head_dim]
  const int32_t* block_tables;  // [B, max_blocks]
  const int32_t* context_lens;  // [B]
  const int32_t* query_start;   // [B + 1]
  int num_seqs;
  int max_blocks;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int head_dim;  // 64 or 128
  int block_size;
  int num_blocks;
  float scale_log2;
  int* status;
  int min_qlen;  // sequences with fewer query rows belong to the other kernels
  // Stream-K pieces: two (O, m, l) slots per CTA, each [256 rows][132 floats],
  // and one count per (item, row), zero between calls.
  float* partials;
  int* counters;
  int dep_at_end;  // 1: launched beside the decode kernel; wait for the grid before at the end
};

// Workspace of the chunk kernel's pieces for a batch of at most
// num_query_tokens rows, and its carving (after the rows kernel's part).
size_t chunk_workspace_bytes(int num_query_tokens, int num_seqs_bound, int num_kv_heads, int group, int num_sms);
void chunk_workspace_layout(void* ws, int num_query_tokens, int num_seqs_bound, int num_kv_heads, int group,
                            int num_sms, ChunkParams* p);

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn();
// [num_blocks, Hkv, block_size, 128] bf16 as a 4-D tensor; box = 64 columns x 16 rows of one (block, head).
int encode_kv16_tmap(CUtensorMap* map, const void* cache, int num_blocks, int num_kv_heads, int block_size,
                     int head_dim, EncodeTiledFn fn);

struct DeviceInfo {
  int num_sms;
};

// The current device's SM count; makes the device's primary context current
// first if the calling host thread has no current context.
int device_info(DeviceInfo* info);
int ensure_context(int dev);
int encode_kv_tmap(CUtensorMap* map, const void* cache, int num_blocks, int num_kv_heads, int block_size,
                   int head_dim);

// Each returns a pa_status.
int launch_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache, const int32_t* slot_mapping,
                  int num_tokens, int num_blocks, int num_kv_heads, int head_dim, int block_size, int* dev_status,
                  cudaStream_t stream, int num_sms);
int launch_append_fp8(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                      const int32_t* slot_mapping, int num_tokens, int num_blocks, int num_kv_heads, int head_dim,
                      int block_size, float k_inv, float v_inv, int* dev_status, cudaStream_t stream, int num_sms);
// ctas > 0: launch that many 8-warp CTAs (one per SM) instead of filling the
// GPU, leaving the other SMs to a kernel launched beside it (head_dim 128).
int launch_rows(const RowsParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, int head_dim,
                cudaStream_t stream, int num_sms, int ctas = 0);
// Workspace of the rows kernel for at most num_rows query rows on a device with
// num_sms SMs, and the carving of a buffer of that size into RowsParams.
// max_keys bounds the keys of any row (max_blocks_per_seq * block_size).
size_t rows_workspace_bytes(int num_rows, int num_q_heads, int num_kv_heads, int head_dim, long long max_keys,
                            int num_sms);
void rows_workspace_layout(void* ws, int num_rows, int num_q_heads, int num_kv_heads, int head_dim,
                           long long max_keys, int num_sms, RowsParams* p);
int rows_supported(int group, int head_dim);
int chunk_supported(int group, int head_dim);
// ctas: CTAs of the launch (one per SM), at most num_sms.
int launch_chunk(const ChunkParams& p, const void* q, const void* k_cache, const void* v_cache, int total_q_tokens,
                 cudaStream_t stream, int num_sms, int ctas);
int cascade_supported(int group, int head_dim);
size_t cascade_partials_bytes(int num_seqs, int num_q_heads, int head_dim);
int launch_cascade(const CascadeParams& p, const void* q, const void* k_cache, const void* v_cache,
                   int total_q_tokens, int head_dim, cudaStream_t stream, int num_sms);
// Host plan of a varlen batch (the words of pa_plan).
enum PlanWord {
  PLAN_MAGIC = 0,    // PLAN_MAGIC_VALUE once filled in
  PLAN_FLAGS,        // PLAN_VERIFY32 | PLAN_VERIFY64 | PLAN_CHUNK | PLAN_ROWS: kernels that have work
  PLAN_DECODE_CTAS,  // > 0: decode rows on this many SMs beside the chunk kernel on the others
  PLAN_NUM_SMS,      // SM count the split was made for
  PLAN_NUM_SEQS,
  PLAN_TOTAL_Q,
  PLAN_GROUP,
  PLAN_HEAD_DIM,
};
constexpr int32_t PLAN_MAGIC_VALUE = 0x50414e31;  // "PAN1"
constexpr int32_t PLAN_VERIFY32 = 1, PLAN_VERIFY64 = 2, PLAN_CHUNK = 4, PLAN_ROWS = 8;

// What a calibration run of the decode kernel overrides.
struct RowsOverride {
  unsigned long long* trace;  // RowsParams::trace
  int weighted;               // -1: the recorded rates, 0: equal split, 1: the rates below
  const uint16_t* sm_rate;
};

// Argument checks, tensor maps and kernel dispatch shared by the attention
// entry points (query_start == nullptr: one query row per sequence).
int run_attention(void* out, const void* q, const int32_t* query_start, const void* k_cache, const void* v_cache,
                  const int32_t* block_tables, int max_blocks, const int32_t* context_lens, int num_seqs,
                  int total_q_tokens, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                  int num_blocks, float scale, void* workspace, size_t workspace_bytes, int* dev_status,
                  void* stream, const void* k_new = nullptr, const void* v_new = nullptr,
                  const int32_t* group_start = nullptr, const int32_t* group_prefix = nullptr, int num_groups = 0,
                  int kv_fp8 = 0, float k_scale = 1.f, float v_scale = 1.f, const int32_t* plan = nullptr,
                  const RowsOverride* ovr = nullptr);
// Bytes of workspace a decode call (one query row per sequence) needs: the
// rows kernel's part of pa_workspace_bytes.
size_t decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                              int block_size);

}  // namespace pa
