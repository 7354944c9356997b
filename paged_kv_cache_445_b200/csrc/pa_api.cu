// pa_api.cu -- the C ABI of libpa.so: argument checks, tensor maps, workspace
// layout and dispatch to the kernels.  See include/pa.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "pa_internal.h"

namespace pa {

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

int device_info(DeviceInfo* info) {
  static PerDevice sms;
  return per_device(
      sms,
      [](int dev) {
        int n = 0;
        return cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n
                                                                                                       : PA_ERR_CUDA;
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
  return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
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
  return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
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

int run_attention(void* out, const void* q, const int32_t* query_start, const void* k_cache,
                         const void* v_cache, const int32_t* block_tables, int max_blocks,
                         const int32_t* context_lens, int num_seqs, int total_q_tokens, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                         void* workspace, size_t workspace_bytes, int* dev_status, void* stream,
                         const void* k_new, const void* v_new, const int32_t* group_start,
                         const int32_t* group_prefix, int num_groups, int kv_fp8, float k_scale, float v_scale) {
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
  if (workspace_bytes < rows_bytes + casc_bytes) return PA_ERR_WORKSPACE;

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
  if (query_start && !kv_fp8 && chunk_supported(p.group, head_dim)) {
    // sequences with 2 .. 64/G query rows run on the tcgen05 multi-row kernel,
    // longer ones on the tcgen05 chunk kernel, the single rows (decodes) on the
    // rows kernel after both
    const bool verify = verify_supported(p.group, head_dim, num_seqs);
    if (verify) {
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
      if ((rc = launch_verify(v, q, k_cache, v_cache, total_q_tokens, st, di.num_sms)) != PA_OK) return rc;
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
    c.block_size = block_size;
    c.num_blocks = num_blocks;
    c.scale_log2 = p.scale_log2;
    c.status = dev_status;
    if ((rc = launch_chunk(c, q, k_cache, v_cache, total_q_tokens, st, di.num_sms)) != PA_OK) return rc;
    p.skip_multi = 1;
  }
  return launch_rows(p, tmk, tmv, head_dim, st, di.num_sms);
}

}  // namespace pa

extern "C" {

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
  return pa::workspace_needed(num_query_tokens, num_q_heads, num_kv_heads, head_dim,
                              static_cast<long long>(max_blocks_per_seq) * block_size, di.num_sms);
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
