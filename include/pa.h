/*
 * pa.h -- C ABI of libpa.so: attention over a paged KV cache on NVIDIA B200 (sm_100a).
 *
 * The KV cache of one attention layer is a pool of fixed-size physical blocks
 * of 16 or 32 tokens.  Each sequence has a block table that maps its logical
 * token positions to physical block IDs; blocks are taken as a sequence grows
 * and may be shared by several sequences ("vLLM serving internals", AI
 * Engineering from Scratch, Phase 17 / 04, section "PagedAttention as a
 * virtual memory system"; "Inference optimization", Phase 10 / 12, section
 * "Paged attention").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is CUDA device memory owned by the caller.  The
 *    library never allocates, frees or synchronises; each call enqueues its
 *    kernels on `stream` (a cudaStream_t, NULL = the legacy default stream)
 *    and returns.  Calls are stateless and thread-safe (pa_decode_static_scratch
 *    is the one exception: see its comment).
 *  - Layouts (row-major, no padding):
 *      q, out        bf16  [num_q_tokens, num_q_heads, head_dim]
 *      k_new, v_new  bf16  [num_tokens, num_kv_heads, head_dim]
 *      k_cache,
 *      v_cache       bf16  [num_blocks, num_kv_heads, block_size, head_dim]
 *      block_tables  int32 [num_seqs, max_blocks_per_seq]   (unused entries: any value, e.g. -1)
 *      context_lens  int32 [num_seqs]   tokens of each sequence INCLUDING this step's new ones
 *      query_start   int32 [num_seqs + 1]  query rows of sequence s are query_start[s] .. query_start[s+1]-1
 *      slot_mapping  int32 [num_tokens]    slot = block_id * block_size + offset; negative = padding
 *  - Supported shapes: head_dim in {64, 128, 256}; block_size in {16, 32};
 *    num_q_heads a multiple of num_kv_heads with group = num_q_heads /
 *    num_kv_heads <= 16 (<= 8 when head_dim = 256).  Query head h reads KV head
 *    h / group.  Pointers must be 16-byte aligned.
 *  - Errors the host can see (null pointer, bad shape, workspace too small)
 *    are returned before anything is launched.  A launch failure returns
 *    PA_ERR_CUDA.  Data-dependent faults (a block ID outside [0, num_blocks),
 *    a context longer than the block table, a slot outside the pool, a wait
 *    that gave up) are detected on the device: if `dev_status` is non-NULL
 *    the kernel ORs the matching PA_ERR_* magnitude bit (see PA_STATUS_BIT)
 *    into *dev_status and the offending access is skipped or reads zeros.
 *    Nothing traps.
 *  - Attention uses bf16 inputs, fp32 accumulation and a bf16 output rounded
 *    to nearest even.  A row whose context is empty produces zeros.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_NULL = -1,        /* a required pointer is NULL */
  PA_ERR_SHAPE = -2,       /* inconsistent or negative sizes */
  PA_ERR_UNSUPPORTED = -3, /* head_dim / block_size / group outside the supported set */
  PA_ERR_WORKSPACE = -4,   /* workspace smaller than pa_workspace_bytes() */
  PA_ERR_RANGE = -5,       /* device: block ID, slot or context outside its table or pool */
  PA_ERR_CUDA = -6,        /* a CUDA runtime or driver call failed */
  PA_ERR_TIMEOUT = -7      /* device: a bounded wait gave up */
} pa_status;

/* Bit that a kernel ORs into *dev_status for device-detected error `code`. */
#define PA_STATUS_BIT(code) (1 << (-(code)))

/*
 * pa_cache_append -- write this step's new K/V rows into their cache slots.
 *
 * Defined by "Inference optimization", section "Build it -- Step 1: a KV
 * cache from scratch" (the new keys and values of a step are stored at the
 * sequence's current length before attention reads the cache), in the paged
 * form of "vLLM serving internals", "PagedAttention as a virtual memory
 * system" (the position lands in the block the table gives).
 *
 * For every token t with slot_mapping[t] >= 0 and every KV head h:
 *   k_cache[slot / block_size, h, slot % block_size, :] = k_new[t, h, :]   (and v likewise)
 * A bit-exact copy.  Negative slots are skipped.  A slot >= num_blocks *
 * block_size is skipped and reported through dev_status.  Two tokens mapped
 * to the same slot race (the caller's allocator never does that).
 */
PA_API int pa_cache_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                    const int32_t* slot_mapping, int num_tokens, int num_blocks, int num_kv_heads,
                    int head_dim, int block_size, int* dev_status, void* stream);

/*
 * pa_workspace_bytes -- bytes of device workspace pa_decode / pa_prefill_chunk
 * need for a batch with at most `num_query_tokens` query rows whose block
 * tables are `max_blocks_per_seq` wide, on the CURRENT device (the figure
 * depends on its SM count).  Returns 0 for invalid sizes.
 *
 * It covers every call the batch may take: at head_dim 64 or 128 with a group
 * the tcgen05 chunk kernel supports it includes that kernel's piece area
 * (two slots of 256 rows x 132 floats per SM, about 40 MB on a 148-SM GPU),
 * which decode calls do not use.
 *
 * Workspace contract: the caller allocates it and ZERO-FILLS it once before
 * its first use; it may then reuse it for any later call on the same stream.
 * The library keeps its counters in it and every call that returns PA_OK and
 * whose dev_status stays clear puts them back to zero; the rest is scratch.
 * Calls that overlap in time must use different workspaces.  After a call
 * that reported a device error, zero it again.
 */
PA_API size_t pa_workspace_bytes(int num_query_tokens, int num_q_heads, int num_kv_heads, int head_dim,
                                 int max_blocks_per_seq, int block_size);

/*
 * pa_decode -- one decode step: each sequence has exactly one query row (the
 * newest token, position context_lens[s] - 1) that attends to all of its
 * cached keys 0 .. context_lens[s] - 1.
 *
 * Defined by "Inference optimization", section "KV cache" (token N computes
 * its own K, V and reads those of tokens 1..N-1 from the cache) and section
 * "Build it -- Step 2: attention with the KV cache" (softmax of the scaled
 * scores with the maximum subtracted, normalised, times V); the keys are
 * gathered through the block table ("PagedAttention as a virtual memory
 * system").  GQA: query head h uses KV head h / (num_q_heads / num_kv_heads)
 * ("Inference optimization", exercise on grouped-query attention).
 *
 *   out[s, h, :] = sum_j softmax_j(scale * q[s, h, :] . K_j) V_j,  j < context_lens[s]
 *
 * q / out have num_seqs rows.  `scale` is usually 1/sqrt(head_dim).  Call
 * pa_cache_append first if this step's rows must be visible.
 */
PA_API int pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
              const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
              int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
              int num_blocks, float scale, void* workspace, size_t workspace_bytes, int* dev_status,
              void* stream);

/*
 * pa_decode_append -- pa_cache_append of this step's rows followed by
 * pa_decode, in one launch.  Row s of k_new / v_new ([num_seqs, num_kv_heads,
 * head_dim] bf16) is the newest token of sequence s; it is written to
 * position context_lens[s] - 1 through the block table (the slot the host
 * allocator hands out for that token), and the attention uses it as that
 * position's key and value.  Output and cache contents are bit-identical to
 * the two separate calls with slot_mapping[s] = that slot.
 *
 * The pages describe the step as one fused call over the batch ("vLLM serving
 * internals", "What the scheduler looks like") and the cache update as part
 * of attention ("Inference optimization", "Build it -- Step 2": the layer
 * stores the new keys and values, then attends over the cache).  Fusing saves
 * the append's launch and lets its stores overlap the attention's loads.
 *
 * k_cache / v_cache are written.  A block ID outside the pool skips that
 * store and sets the RANGE bit; everything else as pa_decode.
 */
PA_API int pa_decode_append(void* out, const void* q, const void* k_new, const void* v_new, void* k_cache,
                            void* v_cache, const int32_t* block_tables, int max_blocks_per_seq,
                            const int32_t* context_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                            int head_dim, int block_size, int num_blocks, float scale, void* workspace,
                            size_t workspace_bytes, int* dev_status, void* stream);

/*
 * FP8 (E4M3) KV cache.  The pages serve the 70B model in FP8 ("vLLM serving
 * internals", introduction and "Numbers to remember"; "How vLLM gets real
 * throughput on H100s", "Hopper-specific tunings") without fixing a format;
 * the cache here stores codes of the OCP 8-bit floating point E4M3 format
 * ("FN" variant: no infinities, largest finite 448) with one scale per
 * tensor: code = E4M3(x * fl32(1 / scale)) (binary32 product, nearest-even,
 * saturated to +-448), value = E4M3value * scale.  k_cache / v_cache are
 * uint8 [num_blocks, num_kv_heads, block_size, head_dim]: half the bytes of
 * bf16, so a decode step reads half the bytes.
 *
 * pa_cache_append_fp8 -- pa_cache_append into an FP8 cache (quantising).
 * Scales must be positive and finite (PA_ERR_SHAPE otherwise).
 */
PA_API int pa_cache_append_fp8(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                               const int32_t* slot_mapping, int num_tokens, int num_blocks, int num_kv_heads,
                               int head_dim, int block_size, float k_scale, float v_scale, int* dev_status,
                               void* stream);

/*
 * pa_decode_fp8 -- pa_decode over an FP8 cache; with k_new / v_new set (both
 * or neither) the step's append is fused in, as in pa_decode_append (the new
 * rows are quantised exactly as pa_cache_append_fp8 does).  q and out stay
 * bf16.  Keys and values enter the tensor cores as f16 (exact for E4M3
 * values) with q converted to f16; accumulation is fp32.  Supported:
 * head_dim 128 or 256 (PA_ERR_UNSUPPORTED otherwise); same workspace as
 * pa_decode.
 */
PA_API int pa_decode_fp8(void* out, const void* q, const void* k_new, const void* v_new, void* k_cache,
                         void* v_cache, const int32_t* block_tables, int max_blocks_per_seq,
                         const int32_t* context_lens, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                         int block_size, int num_blocks, float scale, float k_scale, float v_scale, void* workspace,
                         size_t workspace_bytes, int* dev_status, void* stream);

/*
 * pa_prefill_chunk_fp8 -- pa_prefill_chunk over an FP8 (E4M3) cache, with the
 * scales and code format of pa_decode_fp8: a varlen batch of prefill chunks,
 * verification rows and decodes.  Every row runs on the decode kernel's E4M3
 * path (each row of a sequence reads its keys; the tcgen05 chunk and
 * verification kernels take bf16 caches only), so a long chunk costs one
 * pass over its keys per row.  head_dim 128 or 256; workspace as for
 * pa_prefill_chunk.
 */
PA_API int pa_prefill_chunk_fp8(void* out, const void* q, const int32_t* query_start, const void* k_cache,
                                const void* v_cache, const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* context_lens, int num_seqs, int total_q_tokens, int num_q_heads,
                                int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                                float k_scale, float v_scale, void* workspace, size_t workspace_bytes, int* dev_status,
                                void* stream);

/*
 * pa_decode_cascade -- pa_decode (optionally fused with the append, as
 * pa_decode_append) for a batch in which groups of sequences share a prefix of
 * the KV cache, as copy-on-write forks of one prompt do ("vLLM serving
 * internals", "PagedAttention as a virtual memory system": shared pages are
 * stored once; "How vLLM gets real throughput on H100s", "PagedAttention
 * borrows from operating systems": GRPO rollouts of one prompt share its
 * pages).  The result equals pa_decode's up to rounding: softmax over keys
 * 0..p splits exactly into the shared prefix and the rest.
 *
 * Groups: sequences group_start[g] .. group_start[g+1] - 1 (consecutive;
 * group_start increasing, int32 [num_groups + 1], device) share their first
 * group_prefix[g] tokens (int32 [num_groups], device): those entries of their
 * block tables are identical.  Sequences outside [group_start[0],
 * group_start[num_groups]) are plain decodes.  The first
 * floor(group_prefix[g] / 64) * 64 keys of a group are read once for all its
 * sequences and heads on the tcgen05 tensor cores; each sequence's remaining
 * keys go through the decode kernel, which folds the prefix results in.  Each
 * member's context must extend past that span (PA_ERR_RANGE on the device
 * otherwise).  k_new / v_new: both NULL (append done elsewhere) or both set
 * (fused append as in pa_decode_append).
 *
 * The workspace must hold pa_cascade_workspace_bytes() bytes, zero-filled
 * once (contract of pa_workspace_bytes).  Supported: group <= 128 query heads
 * per KV head, head_dim in {64, 128, 256}.
 */
PA_API size_t pa_cascade_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                         int max_blocks_per_seq, int block_size);
PA_API int pa_decode_cascade(void* out, const void* q, const void* k_new, const void* v_new, void* k_cache,
                             void* v_cache, const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* context_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                             int head_dim, int block_size, int num_blocks, float scale, const int32_t* group_start,
                             const int32_t* group_prefix, int num_groups, void* workspace, size_t workspace_bytes,
                             int* dev_status, void* stream);

/*
 * pa_prefill_chunk -- attention for a varlen batch that mixes prefill chunks
 * and decodes in one call.  Sequence s contributes qlen = query_start[s+1] -
 * query_start[s] query rows: the LAST qlen positions of its context_lens[s]
 * tokens (a chunk of a long prompt, or qlen = 1 for a decode).  Row i of
 * sequence s sits at position p = context_lens[s] - qlen + i and attends
 * causally to keys 0 .. p.
 *
 * Defined by "vLLM serving internals", section "Chunked prefill protects the
 * TTFT tail" (a long prompt is processed in ~512-token chunks interleaved with
 * decodes) and section "What the scheduler looks like" (prefill chunks and
 * single decode tokens form one batch and one fused GPU call); the causal mask
 * of a query block that ends at the last key is the one of "Inference
 * optimization", "Build it -- Step 2" (row i sees keys j <= i + Lk - Lq).
 *
 * q / out have total_q_tokens = query_start[num_seqs] rows.  At head_dim 128
 * (query heads per KV head G in {1, 2, 4, 8, 16}) the call runs, one after
 * another on `stream`: a tcgen05 kernel for sequences with 2 .. 64/G rows
 * (speculative verification: the "Speculative decoding" section of
 * "Inference optimization"; batches of at most 512 sequences), the tcgen05
 * chunk kernel for longer chunks, and the decode path for qlen = 1.  At
 * head_dim 64 with those groups, and at head_dim 64 or 128 with G = 6 or 12,
 * the tcgen05 chunk kernel takes every sequence of 2 or more rows.  Other
 * head dims and groups run every row on the decode path.  A row with no key (p < 0)
 * produces zeros.  Workspace: pa_workspace_bytes(total_q_tokens, ...), under
 * its contract (zero-filled once; the call leaves its counters at zero).
 */
PA_API int pa_prefill_chunk(void* out, const void* q, const int32_t* query_start, const void* k_cache,
                     const void* v_cache, const int32_t* block_tables, int max_blocks_per_seq,
                     const int32_t* context_lens, int num_seqs, int total_q_tokens, int num_q_heads,
                     int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                     void* workspace, size_t workspace_bytes, int* dev_status, void* stream);

/*
 * pa_plan_batch / pa_prefill_chunk_planned -- pa_prefill_chunk with a plan
 * made on the host from host copies of query_start and context_lens (the
 * scheduler that builds a batch has them before it copies them to the
 * device).  The plan records which of the call's kernels have work, so that
 * only those are launched, and, for a batch that mixes decode rows with
 * prefill chunks ("vLLM serving internals", "Chunked prefill protects the
 * TTFT tail" and "What the scheduler looks like": the scheduler's one batch
 * per step), how the GPU's SMs are shared: the decode rows, bound by HBM,
 * stream on some SMs while the tcgen05 chunk kernel, bound by the tensor
 * cores, computes on the others, both at once.  Results equal
 * pa_prefill_chunk's up to rounding (the same definition; a chunk item cut
 * between SMs is merged from its pieces).
 *
 * pa_plan_batch: query_start [num_seqs + 1] and context_lens [num_seqs] are
 * HOST arrays (int32) with the values the device arrays will hold; the other
 * sizes are those of the pa_prefill_chunk call.  Make the plan with the
 * device current that will run the call (it records its SM count).  Returns
 * PA_ERR_NULL / PA_ERR_SHAPE / PA_ERR_UNSUPPORTED for bad arguments.
 *
 * pa_prefill_chunk_planned: the arguments of pa_prefill_chunk plus the plan.
 * A plan whose batch shape (num_seqs, total_q_tokens, group, head_dim) or SM
 * count differs from the call's is rejected with PA_ERR_SHAPE.  A plan that
 * does not match the device arrays' values leaves rows unwritten or
 * misassigned: the caller keeps the two in step.  Workspace as for
 * pa_prefill_chunk.
 */
#define PA_PLAN_WORDS 16
typedef struct pa_plan {
  int32_t words[PA_PLAN_WORDS];
} pa_plan;
PA_API int pa_plan_batch(const int32_t* query_start, const int32_t* context_lens, int num_seqs, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, pa_plan* plan);
PA_API int pa_prefill_chunk_planned(void* out, const void* q, const int32_t* query_start, const void* k_cache,
                                    const void* v_cache, const int32_t* block_tables, int max_blocks_per_seq,
                                    const int32_t* context_lens, int num_seqs, int total_q_tokens, int num_q_heads,
                                    int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                                    void* workspace, size_t workspace_bytes, const pa_plan* plan, int* dev_status,
                                    void* stream);

/*
 * pa_decode_static_scratch -- pa_decode without a caller workspace.  Same
 * arguments, layouts, result and errors as pa_decode, minus `workspace` and
 * `workspace_bytes`.  The sources this library follows describe no such call:
 * it exists for callers that cannot hand the library device memory when they
 * launch (a runtime that may not call the allocator while it replays a
 * recorded sequence of launches, or a host with a fixed memory budget).
 *
 * Scratch: a library-owned device array of PA_STATIC_SCRATCH_BYTES per device
 * (64 MiB), part of the library's device image, so this call allocates
 * nothing.  A batch whose decode workspace (the part of pa_workspace_bytes a
 * decode call uses; pa_workspace_bytes also counts the prefill kernels'
 * part) exceeds that size is rejected with PA_ERR_WORKSPACE before any
 * launch (for example, 8 query heads per KV head at head_dim 128 on a 148-SM
 * B200 fits about 1,570 sequences with 512-block tables).
 *
 * Sharing: every call on a device uses the same array.  Calls that overlap in
 * time on one device (other streams, other host threads) race on it and give
 * wrong results: serialise them.  The array keeps what the previous call
 * left; each call clears the part that must start at zero on `stream` before
 * its kernel, so a call after a failed one needs no reset.
 *
 * Set-up: the first call on a device, with that device current, looks up the
 * array's device address (which may load the library's device code there).
 * Make that first call before any stream capture on that device.  The address
 * is kept per device with the identity of the CUDA context it belongs to;
 * after a device reset (a new primary context) the next call looks it up
 * again, so it too should come before any capture.
 *
 * An empty batch (num_seqs = 0) goes through exactly pa_decode's checks and
 * launches nothing.
 */
#define PA_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)
PA_API int pa_decode_static_scratch(void* out, const void* q, const void* k_cache, const void* v_cache,
                                    const int32_t* block_tables, int max_blocks_per_seq,
                                    const int32_t* context_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                                    int head_dim, int block_size, int num_blocks, float scale, int* dev_status,
                                    void* stream);

/*
 * pa_calibrate -- per-SM shares for the decode kernel's split of the work,
 * measured once on this device.
 *
 * The decode path is bound by HBM bandwidth and hands every warp a fixed
 * contiguous share of the batch's key tiles before it starts (no claims at
 * run time, so results do not depend on timing).  The SMs of a B200 do not
 * stream equally fast under a full load (timed per warp: pairs of SMs at
 * about 44, 51 and 59 GB/s, the same from launch to launch), so with equal
 * shares the GPU waits for its slowest SMs.  pa_calibrate runs the decode
 * kernel on a synthetic batch (128 sequences x 2048 tokens, 64 query / 8 KV
 * heads, head_dim 128) held in `buffer`, times every SM's share, and adjusts
 * per-SM weights over four rounds until the SMs finish together.  Later
 * launches of the kernel variant that was timed (bf16 cache, head_dim 128, up
 * to 8 query heads per KV head, spread over the whole GPU: pa_decode,
 * pa_decode_append, pa_decode_cascade's private keys and the decode rows of
 * an unplanned pa_prefill_chunk on such shapes) give each SM a share in
 * proportion to its weight; the other variants keep equal shares (the
 * weights made them slower).  Not part of the pages' problem statement: a
 * B200 scheduling aid.
 *
 * buffer: device memory of at least pa_calibrate_bytes() bytes (about
 * 1.1 GB; 256-byte aligned), overwritten.  The call WAITS for its own work
 * (the library's one synchronising call: a set-up step, about 20 ms).  Call
 * it once per device, with nothing else running on the device, before the
 * decode calls that should use it; decode calls that overlap it on other
 * host threads keep the split they started with.  Results of decode calls
 * before and after it differ in rounding (the split moves the places where
 * partial sums are cut).  Returns PA_ERR_WORKSPACE for a small buffer,
 * PA_ERR_UNSUPPORTED on a GPU with more than 160 SMs, PA_ERR_RANGE if some
 * SM got no work to time (the equal split stays).
 *
 * pa_calibration -- the recorded weights of the current device (relative,
 * largest 60000; one per SM; weights_out may be NULL): PA_ERR_RANGE if none.
 * pa_calibration_clear -- forget every device's weights (equal split again).
 */
PA_API size_t pa_calibrate_bytes(void);
PA_API int pa_calibrate(void* buffer, size_t bytes, int* dev_status, void* stream);
PA_API int pa_calibration(int* num_sms, uint16_t* weights_out);
PA_API void pa_calibration_clear(void);

/* Human-readable name of a pa_status value (static storage). */
PA_API const char* pa_status_string(int status);

/*
 * The CUDA failure behind the last PA_ERR_CUDA returned on the calling host
 * thread: pa_last_cuda_error() gives its cudaError_t (or, for the driver's
 * tensor-map encoder, CUresult) value, 0 if no call on this thread failed;
 * pa_last_cuda_error_string() names the failing call and the error
 * (thread-local storage, "" if none).  A launch that reports an error left by
 * an earlier kernel that faulted (a sticky error such as an illegal address)
 * names that error.  Not part of the pages' problem statement: diagnostics.
 */
PA_API int pa_last_cuda_error(void);
PA_API const char* pa_last_cuda_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
