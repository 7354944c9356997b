// pa_api.cu -- the C ABI of libpa.so: argument checks, tensor maps, workspace
// layout and dispatch to the kernels.  See include/pa.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <mutex>

#include "pa_internal.h"

namespace pa {

namespace {
thread_local int t_cuda_error = 0;
thread_local char t_cuda_error_text[192] = "";
}  // namespace

int cuda_fail(cudaError_t e, const char* call) {
  t_cuda_error = static_cast<int>(e);
  snprintf(t_cuda_error_text, sizeof t_cuda_error_text, "%s: %s (%s)", call, cudaGetErrorName(e),
           cudaGetErrorString(e));
  return PA_ERR_CUDA;
}

int cu_fail(CUresult r, const char* call) {
  t_cuda_error = static_cast<int>(r);
  snprintf(t_cuda_error_text, sizeof t_cuda_error_text, "%s: CUresult %d", call, static_cast<int>(r));
  return PA_ERR_CUDA;
}

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }



}  // namespace

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}
}  // namespace

// A host thread that has made no CUDA runtime call yet has no current
// context, and the driver's tensor-map encoder then fails.  Make the current
// device's primary context current in that case (cudaSetDevice does so); a
// context the caller made current itself is left alone.
int ensure_context(int dev) {
  CtxGetCurrentFn get = ctx_get_current_fn();
  CUcontext ctx = nullptr;
  if (get && get(&ctx) == CUDA_SUCCESS && ctx != nullptr) return PA_OK;
  const cudaError_t e = cudaSetDevice(dev);
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "cudaSetDevice");
}

int device_info(DeviceInfo* info) {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const int rc = ensure_context(dev);
  if (rc != PA_OK) return rc;
  static PerDevice sms;
  return per_device(
      sms,
      [](int dev) {
        int n = 0;
        const cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        return n > 0 ? n : static_cast<int>(PA_ERR_CUDA);
      },
      &info->num_sms);
}

// [num_blocks, Hkv, block_size, D] bf16 viewed as a 5-D tensor
// (64 columns, block_size rows, D/64 column groups, Hkv, num_blocks): the
// column groups get their own dimension (stride 128 bytes) so that one box
// (64 x 16 x D/64) brings a whole 16-key tile of one (block, head) into shared
// memory as D/64 swizzled [16 x 128-byte] panels, in a single TMA instruction.
int encode_kv_tmap(CUtensorMap* map, const void* cache, int num_blocks, int num_kv_heads, int block_size,
                   int head_dim) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return PA_ERR_CUDA;
  const cuuint64_t row = static_cast<cuuint64_t>(head_dim) * 2;
  const cuuint64_t dims[5] = {64, static_cast<cuuint64_t>(block_size), static_cast<cuuint64_t>(head_dim / 64),
                              static_cast<cuuint64_t>(num_kv_heads), static_cast<cuuint64_t>(num_blocks)};
  const cuuint64_t strides[4] = {row, 128, row * block_size, row * block_size * num_kv_heads};
  const cuuint32_t box[5] = {64, 16, static_cast<cuuint32_t>(head_dim / 64), 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(cache), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : cu_fail(r, "cuTensorMapEncodeTiled");
}

// FP8 cache [num_blocks, Hkv, block_size, D] bytes viewed as (128, block_size,
// D/128, Hkv, num_blocks): one box brings a 16-key tile of one (block, head) as
// D/128 swizzled [16 x 128-byte] panels, the same smem layout as bf16 at half
// the head dim.
static int encode_kv_tmap_fp8(CUtensorMap* map, const void* cache, int num_blocks, int num_kv_heads,
                              int block_size, int head_dim) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return PA_ERR_CUDA;
  const cuuint64_t row = static_cast<cuuint64_t>(head_dim);
  const cuuint64_t dims[5] = {128, static_cast<cuuint64_t>(block_size), static_cast<cuuint64_t>(head_dim / 128),
                              static_cast<cuuint64_t>(num_kv_heads), static_cast<cuuint64_t>(num_blocks)};
  const cuuint64_t strides[4] = {row, 128, row * block_size, row * block_size * num_kv_heads};
  const cuuint32_t box[5] = {128, 16, static_cast<cuuint32_t>(head_dim / 128), 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(cache), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PA_OK : cu_fail(r, "cuTensorMapEncodeTiled");
}

static int check_attention_shape(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                 int num_blocks, int max_blocks) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_blocks <= 0)
    return PA_ERR_SHAPE;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_SHAPE;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (!rows_supported(num_q_heads / num_kv_heads, head_dim)) return PA_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_blocks) * block_size > 0x7fffffffLL) return PA_ERR_SHAPE;
  return PA_OK;
}

static size_t workspace_needed(int num_query_tokens, int num_q_heads, int num_kv_heads, int head_dim,
                               long long max_keys, int num_sms) {
  return rows_workspace_bytes(num_query_tokens, num_q_heads, num_kv_heads, head_dim, max_keys, num_sms);
}

// Multi-row sequences of a batch of num_query_tokens rows: at most half of them.
static int multirow_seq_bound(int num_query_tokens) { return num_query_tokens / 2 + 1; }

// The chunk kernel's piece area, for varlen batches on the tcgen05 path.
static size_t chunk_part(int num_query_tokens, int num_q_heads, int num_kv_heads, int head_dim, int num_sms) {
  const int group = num_q_heads / num_kv_heads;
  if (!chunk_supported(group, head_dim)) return 0;
  return chunk_workspace_bytes(num_query_tokens, multirow_seq_bound(num_query_tokens), num_kv_heads, group, num_sms);
}

int run_attention(void* out, const void* q, const int32_t* query_start, const void* k_cache,
                         const void* v_cache, const int32_t* block_tables, int max_blocks,
                         const int32_t* context_lens, int num_seqs, int total_q_tokens, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                         void* workspace, size_t workspace_bytes, int* dev_status, void* stream,
                         const void* k_new, const void* v_new, const int32_t* group_start,
                         const int32_t* group_prefix, int num_groups, int kv_fp8, float k_scale, float v_scale,
                         const int32_t* plan, const RowsOverride* ovr) {
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !workspace) return PA_ERR_NULL;
  if ((k_new == nullptr) != (v_new == nullptr)) return PA_ERR_NULL;
  if (k_new && query_start) return PA_ERR_UNSUPPORTED;  // the fused append serves one-row (decode) batches
  if (kv_fp8) {  // E4M3 caches: head_dim 128 or 256, no shared-prefix pass, finite positive scales
    if (head_dim != 128 && head_dim != 256) return PA_ERR_UNSUPPORTED;
    if (num_groups > 0) return PA_ERR_UNSUPPORTED;
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !(k_scale < INFINITY) || !(v_scale < INFINITY)) return PA_ERR_SHAPE;
  }
  if (k_new && (!aligned16(k_new) || !aligned16(v_new))) return PA_ERR_SHAPE;
  int rc = check_attention_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks);
  if (rc != PA_OK) return rc;
  if (total_q_tokens < 0) return PA_ERR_SHAPE;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_SHAPE;
  if (num_seqs == 0 || total_q_tokens == 0) return PA_OK;
  DeviceInfo di;
  if ((rc = device_info(&di)) != PA_OK) return rc;
  const long long max_keys = static_cast<long long>(max_blocks) * block_size;
  const size_t rows_bytes =
      (workspace_needed(total_q_tokens, num_q_heads, num_kv_heads, head_dim, max_keys, di.num_sms) + 255) / 256 * 256;
  if (num_groups < 0) return PA_ERR_SHAPE;
  if (num_groups > 0) {  // shared-prefix groups: decode batches only
    if (query_start) return PA_ERR_UNSUPPORTED;
    if (!group_start || !group_prefix) return PA_ERR_NULL;
    if (!cascade_supported(num_q_heads / num_kv_heads, head_dim)) return PA_ERR_UNSUPPORTED;
  }
  const size_t casc_bytes = num_groups > 0 ? cascade_partials_bytes(num_seqs, num_q_heads, head_dim) : 0;
  const bool chunk_path = query_start && !kv_fp8 && chunk_supported(num_q_heads / num_kv_heads, head_dim);
  const size_t chunk_bytes =
      chunk_path ? chunk_part(total_q_tokens, num_q_heads, num_kv_heads, head_dim, di.num_sms) : 0;
  if (workspace_bytes < rows_bytes + casc_bytes + chunk_bytes) return PA_ERR_WORKSPACE;
  if (plan) {  // a plan made for this batch shape on a GPU of this size
    if (plan[PLAN_MAGIC] != PLAN_MAGIC_VALUE || plan[PLAN_NUM_SEQS] != num_seqs ||
        plan[PLAN_TOTAL_Q] != total_q_tokens || plan[PLAN_GROUP] != num_q_heads / num_kv_heads ||
        plan[PLAN_HEAD_DIM] != head_dim || plan[PLAN_NUM_SMS] != di.num_sms)
      return PA_ERR_SHAPE;
  }

  CUtensorMap tmk, tmv;
  if (kv_fp8) {
    if ((rc = encode_kv_tmap_fp8(&tmk, k_cache, num_blocks, num_kv_heads, block_size, head_dim)) != PA_OK) return rc;
    if ((rc = encode_kv_tmap_fp8(&tmv, v_cache, num_blocks, num_kv_heads, block_size, head_dim)) != PA_OK) return rc;
  } else {
    if ((rc = encode_kv_tmap(&tmk, k_cache, num_blocks, num_kv_heads, block_size, head_dim)) != PA_OK) return rc;
    if ((rc = encode_kv_tmap(&tmv, v_cache, num_blocks, num_kv_heads, block_size, head_dim)) != PA_OK) return rc;
  }

  RowsParams p{};
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.query_start = query_start;
  p.num_seqs = num_seqs;
  p.max_blocks = max_blocks;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = num_q_heads / num_kv_heads;
  p.block_size = block_size;
  p.num_blocks = num_blocks;
  p.skip_multi = 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.kv_fp8 = kv_fp8;
  p.v_scale = 1.f;
  p.k_inv_scale = p.v_inv_scale = 1.f;
  if (kv_fp8) {  // scores of codes times k_scale: fold it into the softmax scale
    p.scale_log2 = scale * k_scale * 1.4426950408889634f;
    p.v_scale = v_scale;
    p.k_inv_scale = 1.f / k_scale;
    p.v_inv_scale = 1.f / v_scale;
  }
  rows_workspace_layout(workspace, total_q_tokens, num_q_heads, num_kv_heads, head_dim, max_keys, di.num_sms, &p);
  p.num_sms = di.num_sms;
  p.weighted = di.num_sms <= PA_MAX_WEIGHTED_SMS && sm_rates_snapshot(p.sm_rate, di.num_sms) ? 1 : 0;
  if (ovr) {
    p.trace = ovr->trace;
    if (ovr->weighted == 0) p.weighted = 0;
    if (ovr->weighted == 1 && ovr->sm_rate && di.num_sms <= PA_MAX_WEIGHTED_SMS) {
      p.weighted = 1;
      for (int i = 0; i < di.num_sms; ++i) p.sm_rate[i] = ovr->sm_rate[i];
    }
  }
  if (p.weighted) {  // prefix sums for a whole-GPU launch: each CTA then needs two words
    p.sm_prefix[0] = 0;
    for (int i = 0; i < di.num_sms; ++i) p.sm_prefix[i + 1] = p.sm_prefix[i] + p.sm_rate[i];
  }
  p.status = dev_status;
  p.k_new = k_new;
  p.v_new = v_new;
  p.k_cache = const_cast<void*>(k_cache);
  p.v_cache = const_cast<void*>(v_cache);
  p.group_start = group_start;
  p.group_prefix = group_prefix;
  p.num_groups = num_groups;
  p.casc_partials = num_groups > 0 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + rows_bytes) : nullptr;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (num_groups > 0) {
    // the shared prefixes first: per-slice partials that the rows kernel folds in
    CascadeParams c{};
    c.block_tables = block_tables;
    c.max_blocks = max_blocks;
    c.group_start = group_start;
    c.group_prefix = group_prefix;
    c.num_groups = num_groups;
    c.num_q_heads = num_q_heads;
    c.num_kv_heads = num_kv_heads;
    c.group = p.group;
    c.block_size = block_size;
    c.num_blocks = num_blocks;
    c.scale_log2 = p.scale_log2;
    c.partials = const_cast<float*>(p.casc_partials);
    c.status = dev_status;
    if ((rc = launch_cascade(c, q, k_cache, v_cache, total_q_tokens, head_dim, st, di.num_sms)) != PA_OK) return rc;
  }
  if (chunk_path) {
    // sequences with 2 .. 64/G query rows run on the tcgen05 multi-row kernel,
    // longer ones on the tcgen05 chunk kernel, the single rows (decodes) on the
    // rows kernel.  Without a plan all three are launched (one that finds no
    // work returns at once), one after another on the whole GPU.  With a plan
    // only those with work are, and the decode rows may stream on part of the
    // SMs while the chunk kernel computes on the rest.
    const bool verify = verify_supported(p.group, head_dim, num_seqs);
    int verify_which = verify ? 3 : 0, run_chunk = 1, run_rows = 1, decode_ctas = 0;
    if (plan) {
      verify_which = verify ? (plan[PLAN_FLAGS] & (PLAN_VERIFY32 | PLAN_VERIFY64)) : 0;
      run_chunk = (plan[PLAN_FLAGS] & PLAN_CHUNK) != 0;
      run_rows = (plan[PLAN_FLAGS] & PLAN_ROWS) != 0;
      decode_ctas = plan[PLAN_DECODE_CTAS];
    }
    if (verify_which) {
      VerifyParams v{};
      v.out = out;
      v.block_tables = block_tables;
      v.context_lens = context_lens;
      v.query_start = query_start;
      v.num_seqs = num_seqs;
      v.max_blocks = max_blocks;
      v.num_q_heads = num_q_heads;
      v.num_kv_heads = num_kv_heads;
      v.group = p.group;
      v.block_size = block_size;
      v.num_blocks = num_blocks;
      v.scale_log2 = p.scale_log2;
      v.status = dev_status;
      v.slots = p.partials;
      v.counters = p.verify_counters;
      if ((rc = launch_verify(v, q, k_cache, v_cache, total_q_tokens, st, di.num_sms, verify_which)) != PA_OK)
        return rc;
    }
    ChunkParams c{};
    c.min_qlen = verify ? VERIFY_MAX_COLS / p.group + 1 : 2;
    c.out = out;
    c.block_tables = block_tables;
    c.context_lens = context_lens;
    c.query_start = query_start;
    c.num_seqs = num_seqs;
    c.max_blocks = max_blocks;
    c.num_q_heads = num_q_heads;
    c.num_kv_heads = num_kv_heads;
    c.group = p.group;
    c.head_dim = head_dim;
    c.block_size = block_size;
    c.num_blocks = num_blocks;
    c.scale_log2 = p.scale_log2;
    c.status = dev_status;
    chunk_workspace_layout(static_cast<uint8_t*>(workspace) + rows_bytes, total_q_tokens,
                           multirow_seq_bound(total_q_tokens), num_kv_heads, p.group, di.num_sms, &c);
    p.skip_multi = 1;
    if (run_chunk && run_rows && decode_ctas > 0 && decode_ctas < di.num_sms) {
      // the decode rows first, on decode_ctas SMs; they release the chunk
      // kernel, which takes the other SMs and finishes after them
      p.trigger_early = 1;
      if ((rc = launch_rows(p, tmk, tmv, head_dim, st, di.num_sms, decode_ctas)) != PA_OK) return rc;
      c.dep_at_end = 1;
      return launch_chunk(c, q, k_cache, v_cache, total_q_tokens, st, di.num_sms, di.num_sms - decode_ctas);
    }
    if (run_chunk && (rc = launch_chunk(c, q, k_cache, v_cache, total_q_tokens, st, di.num_sms, di.num_sms)) != PA_OK)
      return rc;
    if (!run_rows) return PA_OK;
  }
  return launch_rows(p, tmk, tmv, head_dim, st, di.num_sms);
}

size_t decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                              int block_size) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads) return 0;
  if (max_blocks_per_seq <= 0 || (block_size != 16 && block_size != 32)) return 0;
  if (!rows_supported(num_q_heads / num_kv_heads, head_dim)) return 0;
  DeviceInfo di;
  if (device_info(&di) != PA_OK) return 0;
  return (workspace_needed(num_seqs, num_q_heads, num_kv_heads, head_dim,
                           static_cast<long long>(max_blocks_per_seq) * block_size, di.num_sms) +
          255) / 256 * 256;
}

namespace {
// Per-SM rates of the kernels on a B200, used only to share the SMs between
// the decode rows and the chunk rows of one batch (measured beside each
// other on the mixed 512-token chunk + 127 decodes batch, where a sweep of
// the split put both sides' end together at 60 decode SMs: an 8-warp decode
// CTA streams about 66 GB/s of KV, the tcgen05 chunk kernel on stream-K
// ranges about 6.0 TFLOP/s per SM; the decode rows of a whole GPU about 6.2
// TB/s).  A split is used when its model time beats running the two kernels
// one after the other on the whole GPU by 5 %.  The decode side takes an
// even number of SMs: SMs come in pairs, and a pair shared by a decode CTA
// and a chunk CTA slowed the step by about 12 % (642 us at 59 and 61 decode
// SMs against 571 and 577 us at 60 and 62).
constexpr double DECODE_BYTES_PER_S_PER_SM = 66e9;
constexpr double DECODE_BYTES_PER_S_ALL = 6.2e12;
constexpr double CHUNK_FLOPS_PER_S_PER_SM = 6.0e12;

int plan_split(double decode_bytes, double chunk_flops, int num_sms) {
  const double serial = decode_bytes / DECODE_BYTES_PER_S_ALL + chunk_flops / (num_sms * CHUNK_FLOPS_PER_S_PER_SM);
  double best = serial;
  int best_n = 0;
  for (int n = 2; n < num_sms; n += 2) {
    const double bw = n * DECODE_BYTES_PER_S_PER_SM < DECODE_BYTES_PER_S_ALL ? n * DECODE_BYTES_PER_S_PER_SM
                                                                             : DECODE_BYTES_PER_S_ALL;
    const double td = decode_bytes / bw, tc = chunk_flops / ((num_sms - n) * CHUNK_FLOPS_PER_S_PER_SM);
    const double t = td > tc ? td : tc;
    if (t < best) {
      best = t;
      best_n = n;
    }
  }
  return best < 0.95 * serial ? best_n : 0;
}
}  // namespace

}  // namespace pa

extern "C" {

int pa_plan_batch(const int32_t* query_start, const int32_t* context_lens, int num_seqs, int num_q_heads,
                  int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, pa_plan* plan) {
  if (!query_start || !context_lens || !plan) return PA_ERR_NULL;
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0) return PA_ERR_SHAPE;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_SHAPE;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  const int group = num_q_heads / num_kv_heads;
  if (!pa::rows_supported(group, head_dim)) return PA_ERR_UNSUPPORTED;
  if (query_start[0] != 0) return PA_ERR_SHAPE;
  pa::DeviceInfo di;
  int rc = pa::device_info(&di);
  if (rc != PA_OK) return rc;
  const bool chunk = pa::chunk_supported(group, head_dim);
  const bool verify = chunk && pa::verify_supported(group, head_dim, num_seqs);
  const int min_qlen = verify ? pa::VERIFY_MAX_COLS / group + 1 : 2;
  const long long cap = static_cast<long long>(max_blocks_per_seq) * block_size;
  int32_t flags = 0;
  double decode_bytes = 0.0, chunk_flops = 0.0;
  for (int s = 0; s < num_seqs; ++s) {
    const long long qlen = static_cast<long long>(query_start[s + 1]) - query_start[s];
    if (qlen < 0) return PA_ERR_SHAPE;
    long long ctx = context_lens[s] < 0 ? 0 : context_lens[s];
    if (ctx > cap) ctx = cap;
    if (qlen == 0) continue;
    if (qlen > ctx) flags |= pa::PLAN_ROWS;  // rows with no key are written as zeros by the rows kernel
    if (!chunk || qlen == 1) {
      flags |= pa::PLAN_ROWS;
      decode_bytes += static_cast<double>(ctx) * num_kv_heads * head_dim * 4.0 * static_cast<double>(qlen);
    } else if (verify && qlen * group <= pa::VERIFY_MAX_COLS) {
      flags |= qlen * group <= 32 ? pa::PLAN_VERIFY32 : pa::PLAN_VERIFY64;
    } else if (qlen >= min_qlen) {
      flags |= pa::PLAN_CHUNK;
      // causal: row i sees ctx - qlen + i + 1 keys
      const double first = static_cast<double>(ctx - qlen + 1);
      const double keys = qlen * first + 0.5 * static_cast<double>(qlen) * static_cast<double>(qlen - 1);
      chunk_flops += keys * num_q_heads * head_dim * 4.0;
    }
  }
  int32_t* w = plan->words;
  for (int i = 0; i < PA_PLAN_WORDS; ++i) w[i] = 0;
  w[pa::PLAN_MAGIC] = pa::PLAN_MAGIC_VALUE;
  w[pa::PLAN_FLAGS] = flags;
  w[pa::PLAN_DECODE_CTAS] =
      (flags & pa::PLAN_CHUNK) && (flags & pa::PLAN_ROWS) ? pa::plan_split(decode_bytes, chunk_flops, di.num_sms) : 0;
  w[pa::PLAN_NUM_SMS] = di.num_sms;
  w[pa::PLAN_NUM_SEQS] = num_seqs;
  w[pa::PLAN_TOTAL_Q] = query_start[num_seqs];
  w[pa::PLAN_GROUP] = group;
  w[pa::PLAN_HEAD_DIM] = head_dim;
  return PA_OK;
}

int pa_prefill_chunk_planned(void* out, const void* q, const int32_t* query_start, const void* k_cache,
                             const void* v_cache, const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* context_lens, int num_seqs, int total_q_tokens, int num_q_heads,
                             int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                             void* workspace, size_t workspace_bytes, const pa_plan* plan, int* dev_status,
                             void* stream) {
  if (!query_start || !plan) return PA_ERR_NULL;
  return pa::run_attention(out, q, query_start, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                           num_seqs, total_q_tokens, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                           scale, workspace, workspace_bytes, dev_status, stream, nullptr, nullptr, nullptr, nullptr,
                           0, 0, 1.f, 1.f, plan->words);
}

int pa_cache_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache, const int32_t* slot_mapping,
                    int num_tokens, int num_blocks, int num_kv_heads, int head_dim, int block_size, int* dev_status,
                    void* stream) {
  if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0) return PA_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping) return PA_ERR_NULL;
  if (!pa::aligned16(k_new) || !pa::aligned16(v_new) || !pa::aligned16(k_cache) || !pa::aligned16(v_cache))
    return PA_ERR_SHAPE;
  pa::DeviceInfo di;
  int rc = pa::device_info(&di);
  if (rc != PA_OK) return rc;
  return pa::launch_append(k_new, v_new, k_cache, v_cache, slot_mapping, num_tokens, num_blocks, num_kv_heads,
                           head_dim, block_size, dev_status, static_cast<cudaStream_t>(stream), di.num_sms);
}

size_t pa_workspace_bytes(int num_query_tokens, int num_q_heads, int num_kv_heads, int head_dim,
                          int max_blocks_per_seq, int block_size) {
  if (num_query_tokens < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads) return 0;
  if (max_blocks_per_seq <= 0 || (block_size != 16 && block_size != 32)) return 0;
  if (!pa::rows_supported(num_q_heads / num_kv_heads, head_dim)) return 0;
  pa::DeviceInfo di;
  if (pa::device_info(&di) != PA_OK) return 0;
  const size_t rows = (pa::workspace_needed(num_query_tokens, num_q_heads, num_kv_heads, head_dim,
                                            static_cast<long long>(max_blocks_per_seq) * block_size, di.num_sms) +
                       255) / 256 * 256;
  return rows + pa::chunk_part(num_query_tokens, num_q_heads, num_kv_heads, head_dim, di.num_sms);
}

int pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
              int max_blocks_per_seq, const int32_t* context_lens, int num_seqs, int num_q_heads, int num_kv_heads,
              int head_dim, int block_size, int num_blocks, float scale, void* workspace, size_t workspace_bytes,
              int* dev_status, void* stream) {
  return pa::run_attention(out, q, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                           num_seqs, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                           workspace, workspace_bytes, dev_status, stream);
}

int pa_decode_append(void* out, const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                     const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                     int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                     void* workspace, size_t workspace_bytes, int* dev_status, void* stream) {
  if (!k_new || !v_new) return PA_ERR_NULL;
  return pa::run_attention(out, q, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                           num_seqs, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                           workspace, workspace_bytes, dev_status, stream, k_new, v_new);
}

size_t pa_cascade_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                  int max_blocks_per_seq, int block_size) {
  const size_t rows = pa_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, block_size);
  if (rows == 0 || !pa::cascade_supported(num_q_heads / num_kv_heads, head_dim)) return 0;
  return (rows + 255) / 256 * 256 + pa::cascade_partials_bytes(num_seqs, num_q_heads, head_dim);
}

int pa_decode_cascade(void* out, const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                      const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                      int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                      const int32_t* group_start, const int32_t* group_prefix, int num_groups, void* workspace,
                      size_t workspace_bytes, int* dev_status, void* stream) {
  if ((k_new == nullptr) != (v_new == nullptr)) return PA_ERR_NULL;
  return pa::run_attention(out, q, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                           num_seqs, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                           workspace, workspace_bytes, dev_status, stream, k_new, v_new, group_start, group_prefix,
                           num_groups);
}

int pa_cache_append_fp8(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                        const int32_t* slot_mapping, int num_tokens, int num_blocks, int num_kv_heads, int head_dim,
                        int block_size, float k_scale, float v_scale, int* dev_status, void* stream) {
  if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0) return PA_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (!(k_scale > 0.f) || !(v_scale > 0.f) || !(k_scale < INFINITY) || !(v_scale < INFINITY)) return PA_ERR_SHAPE;
  if (num_tokens == 0) return PA_OK;
  if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping) return PA_ERR_NULL;
  if (!pa::aligned16(k_new) || !pa::aligned16(v_new) || !pa::aligned16(k_cache) || !pa::aligned16(v_cache))
    return PA_ERR_SHAPE;
  pa::DeviceInfo di;
  int rc = pa::device_info(&di);
  if (rc != PA_OK) return rc;
  return pa::launch_append_fp8(k_new, v_new, k_cache, v_cache, slot_mapping, num_tokens, num_blocks, num_kv_heads,
                               head_dim, block_size, 1.f / k_scale, 1.f / v_scale, dev_status,
                               static_cast<cudaStream_t>(stream), di.num_sms);
}

int pa_decode_fp8(void* out, const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                  const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                  int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                  float k_scale, float v_scale, void* workspace, size_t workspace_bytes, int* dev_status,
                  void* stream) {
  if ((k_new == nullptr) != (v_new == nullptr)) return PA_ERR_NULL;
  return pa::run_attention(out, q, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                           num_seqs, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                           workspace, workspace_bytes, dev_status, stream, k_new, v_new, nullptr, nullptr, 0, 1,
                           k_scale, v_scale);
}

int pa_prefill_chunk_fp8(void* out, const void* q, const int32_t* query_start, const void* k_cache,
                         const void* v_cache, const int32_t* block_tables, int max_blocks_per_seq,
                         const int32_t* context_lens, int num_seqs, int total_q_tokens, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale, float k_scale,
                         float v_scale, void* workspace, size_t workspace_bytes, int* dev_status, void* stream) {
  if (!query_start) return PA_ERR_NULL;
  return pa::run_attention(out, q, query_start, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                           num_seqs, total_q_tokens, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                           scale, workspace, workspace_bytes, dev_status, stream, nullptr, nullptr, nullptr, nullptr,
                           0, 1, k_scale, v_scale);
}

int pa_prefill_chunk(void* out, const void* q, const int32_t* query_start, const void* k_cache, const void* v_cache,
                     const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                     int total_q_tokens, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                     int num_blocks, float scale, void* workspace, size_t workspace_bytes, int* dev_status,
                     void* stream) {
  if (!query_start) return PA_ERR_NULL;
  return pa::run_attention(out, q, query_start, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                           num_seqs, total_q_tokens, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                           scale, workspace, workspace_bytes, dev_status, stream);
}

int pa_last_cuda_error(void) { return pa::t_cuda_error; }

const char* pa_last_cuda_error_string(void) { return pa::t_cuda_error_text; }

const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_NULL: return "PA_ERR_NULL: a required pointer is NULL";
    case PA_ERR_SHAPE: return "PA_ERR_SHAPE: inconsistent sizes or misaligned pointer";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: head_dim, block_size or group outside the supported set";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: workspace smaller than pa_workspace_bytes()";
    case PA_ERR_RANGE: return "PA_ERR_RANGE: block ID, slot or context outside its table or pool";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: a CUDA call failed";
    case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT: a bounded device wait gave up";
    default: return "unknown pa_status";
  }
}

}  // extern "C"
