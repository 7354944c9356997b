// pa_append.cu -- cache append: scatter this step's K/V rows into their slots.
//
// "Inference optimization" (AI Engineering from Scratch, Phase 10 / 12),
// "Build it -- Step 1: a KV cache from scratch": a step's new keys and values
// are stored at the sequence's current length before attention reads the
// cache; in the paged layout the position's slot (block * block_size + offset)
// comes from the block table ("vLLM serving internals", "PagedAttention as a
// virtual memory system").
//
// HBM-bound bit copy.  One 16-byte vector per thread per iteration: a row of
// head_dim bf16 is head_dim / 8 vectors, so consecutive threads read
// consecutive 16-byte pieces of k_new (coalesced) and write whole 128..512-byte
// rows of the cache.
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

__global__ void __launch_bounds__(256) append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                                     uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                                     const int32_t* __restrict__ slot_mapping, int num_tokens,
                                                     int num_kv_heads, int vec_per_row, int block_size,
                                                     long long num_slots, int* status) {
  grid_launch_dependents();  // the attention kernel after this one may start its prologue now
  const long long per_token = static_cast<long long>(num_kv_heads) * vec_per_row;
  const long long total = per_token * num_tokens;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = idx / per_token;
    const long long rem = idx - t * per_token;
    const long long h = rem / vec_per_row;
    const long long v = rem - h * vec_per_row;
    const long long slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (h == 0 && v == 0) set_status(status, PA_STATUS_BIT(PA_ERR_RANGE));
      continue;
    }
    const long long blk = slot / block_size, off = slot - blk * block_size;
    const long long dst = ((blk * num_kv_heads + h) * block_size + off) * vec_per_row + v;
    k_cache[dst] = __ldg(k_new + idx);
    v_cache[dst] = __ldg(v_new + idx);
  }
}

// FP8 (E4M3) cache: each 16-byte vector of 8 bf16 becomes 8 codes of
// value * inv_scale (binary32 product, nearest-even, saturated to +-448).
__device__ __forceinline__ uint32_t e4m3_pair(uint32_t w, float inv) {
  return f32x2_to_e4m3x2(__uint_as_float(w << 16) * inv, __uint_as_float(w & 0xffff0000u) * inv);
}

__global__ void __launch_bounds__(256)
    append_fp8_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint2* __restrict__ k_cache,
                      uint2* __restrict__ v_cache, const int32_t* __restrict__ slot_mapping, int num_tokens,
                      int num_kv_heads, int vec_per_row, int block_size, long long num_slots, float k_inv,
                      float v_inv, int* status) {
  grid_launch_dependents();
  const long long per_token = static_cast<long long>(num_kv_heads) * vec_per_row;
  const long long total = per_token * num_tokens;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = idx / per_token;
    const long long rem = idx - t * per_token;
    const long long h = rem / vec_per_row;
    const long long v = rem - h * vec_per_row;
    const long long slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (h == 0 && v == 0) set_status(status, PA_STATUS_BIT(PA_ERR_RANGE));
      continue;
    }
    const long long blk = slot / block_size, off = slot - blk * block_size;
    const long long dst = ((blk * num_kv_heads + h) * block_size + off) * vec_per_row + v;
    const uint4 kx = __ldg(k_new + idx), vx = __ldg(v_new + idx);
    k_cache[dst] = make_uint2(e4m3_pair(kx.x, k_inv) | (e4m3_pair(kx.y, k_inv) << 16),
                              e4m3_pair(kx.z, k_inv) | (e4m3_pair(kx.w, k_inv) << 16));
    v_cache[dst] = make_uint2(e4m3_pair(vx.x, v_inv) | (e4m3_pair(vx.y, v_inv) << 16),
                              e4m3_pair(vx.z, v_inv) | (e4m3_pair(vx.w, v_inv) << 16));
  }
}

int launch_append_fp8(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                      const int32_t* slot_mapping, int num_tokens, int num_blocks, int num_kv_heads, int head_dim,
                      int block_size, float k_inv, float v_inv, int* dev_status, cudaStream_t stream, int num_sms) {
  const int vec_per_row = head_dim / 8;
  const long long total = static_cast<long long>(num_tokens) * num_kv_heads * vec_per_row;
  if (total == 0) return PA_OK;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  const long long cap = static_cast<long long>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  append_fp8_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint2*>(k_cache),
      static_cast<uint2*>(v_cache), slot_mapping, num_tokens, num_kv_heads, vec_per_row, block_size,
      static_cast<long long>(num_blocks) * block_size, k_inv, v_inv, dev_status);
  return check_launch(cudaSuccess, "append_kernel (fp8) launch");
}

int launch_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache, const int32_t* slot_mapping,
                  int num_tokens, int num_blocks, int num_kv_heads, int head_dim, int block_size, int* dev_status,
                  cudaStream_t stream, int num_sms) {
  const int vec_per_row = head_dim / 8;
  const long long total = static_cast<long long>(num_tokens) * num_kv_heads * vec_per_row;
  if (total == 0) return PA_OK;
  // Ask for the same L1/shared split as the attention kernels that follow,
  // so that the SMs need no reconfiguration between the two launches.
  static PerDevice carveout;
  int done = 0;
  (void)per_device(
      carveout,
      [](int) {
        (void)cudaFuncSetAttribute(append_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                   cudaSharedmemCarveoutMaxShared);
        (void)cudaGetLastError();  // a preference only: a refusal is not an error
        return 1;
      },
      &done);
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  const long long cap = static_cast<long long>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  append_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), slot_mapping, num_tokens, num_kv_heads, vec_per_row, block_size,
      static_cast<long long>(num_blocks) * block_size, dev_status);
  return check_launch(cudaSuccess, "append_kernel launch");
}

}  // namespace pa
