// pa_noalloc.cu -- pa_decode with library-owned scratch, for callers that
// cannot allocate device memory at the moment they launch.
//
// The decode kernel needs a scratch buffer (grid-barrier counters, records of
// the segments whose keys were split between warps, and their partial
// results).  pa_decode takes it from the caller.  Some callers have no way to
// provide one: a runtime that must not call the allocator while it replays a
// recorded launch sequence, or a host that owns a fixed memory budget and
// hands out no further buffers.  This entry point uses a fixed-size array that
// lives in the library's own device image instead, so it allocates nothing.
//
// Rules that follow from sharing one array:
//  * The array is per device, per process, and every call on that device uses
//    the same bytes.  Calls that overlap in time (two streams, two host
//    threads) race on it and give wrong results; serialise them.
//  * The array keeps whatever the previous call left.  Each call first clears
//    the part that must start at zero (barrier counters and segment records)
//    on the caller's stream, so a call that follows a failed one is still
//    correct.
//  * The first call on a device (in each CUDA context of it) looks the array's
//    address up; that may load this file's device code on the device.  Make
//    that first call before any stream capture on that device.  The address is
//    cached per device together with the identity of the context it was taken
//    in: after a device reset the primary context is a new one, its copy of
//    the array may sit at another address, and the next call looks it up again.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "pa_internal.h"

// The scratch array: one copy per device, zero-initialised when this file's
// device code is loaded, never freed.
static __device__ __align__(256) unsigned char g_decode_scratch[PA_STATIC_SCRATCH_BYTES];

namespace pa {
namespace {

constexpr int MAX_DEVICES = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct ScratchAddress {
  unsigned long long ctx_id;  // the context the address belongs to
  void* ptr;                  // nullptr: not looked up yet
};

std::mutex g_setup_mu;
ScratchAddress g_scratch[MAX_DEVICES] = {};

// Unique ID of the calling thread's current CUDA context (IDs are never reused
// within a process, unlike context handles).  Returns false if there is none.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Address of the current device's copy of g_decode_scratch, looked up once per
// (device, context) with that device current.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return PA_ERR_CUDA;
  const int rc = ensure_context(dev);
  if (rc != PA_OK) return rc;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  if (have_id && g_scratch[dev].ptr && g_scratch[dev].ctx_id == id) {
    *out = g_scratch[dev].ptr;
    return PA_OK;
  }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess || p == nullptr) {
    (void)cudaGetLastError();
    return e != cudaSuccess ? cuda_fail(e, "cudaGetSymbolAddress") : static_cast<int>(PA_ERR_CUDA);
  }
  // the lookup makes the device's primary context current if no context was
  unsigned long long id_now = 0;
  if (current_context_id(&id_now)) {
    g_scratch[dev].ctx_id = id_now;
    g_scratch[dev].ptr = p;
  }
  *out = p;
  return PA_OK;
}

}  // namespace
}  // namespace pa

extern "C" int pa_decode_static_scratch(void* out, const void* q, const void* k_cache, const void* v_cache,
                                        const int32_t* block_tables, int max_blocks_per_seq,
                                        const int32_t* context_lens, int num_seqs, int num_q_heads,
                                        int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                        float scale, int* dev_status, void* stream) {
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_NULL;
  if (num_seqs < 0) return PA_ERR_SHAPE;
  const size_t need =
      num_seqs > 0
          ? pa::decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, block_size)
          : 0;
  if (need == 0) {
    // an empty batch or invalid sizes: pa_decode's own checks decide, and
    // they return before any launch and before the workspace is looked at
    static unsigned char dummy[256];
    return pa::run_attention(out, q, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                             num_seqs, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                             scale, dummy, 0, dev_status, stream);
  }
  if (need > PA_STATIC_SCRATCH_BYTES) return PA_ERR_WORKSPACE;
  void* ws = nullptr;
  int rc = pa::scratch_for_current_device(&ws);
  if (rc != PA_OK) return rc;
  // the leading part of the workspace (counters, then segment records, up to
  // the piece table) must read zero when the kernel starts
  pa::RowsParams lay{};
  pa::DeviceInfo di;
  if ((rc = pa::device_info(&di)) != PA_OK) return rc;
  pa::rows_workspace_layout(ws, num_seqs, num_q_heads, num_kv_heads, head_dim,
                            static_cast<long long>(max_blocks_per_seq) * block_size, di.num_sms, &lay);
  const size_t zero_bytes =
      static_cast<size_t>(reinterpret_cast<unsigned char*>(lay.table) - static_cast<unsigned char*>(ws));
  const cudaError_t e = cudaMemsetAsync(ws, 0, zero_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return pa::cuda_fail(e, "cudaMemsetAsync");
  return pa::run_attention(out, q, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                           num_seqs, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                           ws, PA_STATIC_SCRATCH_BYTES, dev_status, stream);
}
