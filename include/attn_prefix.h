/*
 * attn_prefix.h -- C ABI of the B200 (sm_100a) prefix-masked attention forward library.
 *
 * Operation.  Exact scaled-dot-product attention forward where batch element b attends
 * only to its first kv_len[b] keys:
 *
 *     out[b,h,i,:] = sum_{j < kv_len[b]} softmax_j(scale * q[b,h,i,:] . k[b,h,j,:]) v[b,h,j,:]
 *     lse[b,h,i]   = ln sum_{j < kv_len[b]} exp(scale * q[b,h,i,:] . k[b,h,j,:])
 *
 * This is the boolean [B,1,1,Tk] key-prefix padding mask of "Rewrite prefix key-padding
 * masks as k/v truncation to keep SDPA on the flash path" (sections "Problem" and
 * "Fix": masking all but the first n keys equals truncating k/v to n rows), carried
 * per batch element as a count of valid keys like the key_value_seq_lengths of "Add
 * sequence-parallel multi-GPU inference ... and a cuDNN flash attention option"
 * (section "cuDNN flash attention"), and shared by all heads as in "Broadcast SDPA
 * attn_mask instead of materializing a per-head copy" (section "What").  The softmax
 * runs online in fp32 and emits the per-row log-sum-exp, so partial results over
 * disjoint key ranges combine exactly ("Add sequence-parallel ...", section
 * "Sequence-parallel inference"): attn_prefix_fwd_split + attn_lse_combine.
 *
 * Conventions for every entry point:
 *   - Tensor pointers are CUDA device memory owned by the caller.  The library never
 *     allocates, frees or keeps them.  Layout is row-major [B, H, T, D] ("BHTD").
 *   - q, k, v, out are bf16 (IEEE binary16-brain, 2 bytes).  lse and split partials
 *     are fp32.  kv_len is int32 [B] in DEVICE memory; the host never reads it.
 *   - All work is enqueued on `stream` (NULL = legacy default stream); no entry point
 *     synchronizes except attn_get_device_status.
 *   - Arguments are checked on the host before any launch; a failed check returns a
 *     status and enqueues nothing.  Pointers must be 16-byte aligned (TMA rule).
 *   - kv_len[b] outside [0, Tk] is clamped into range inside the kernel and raises the
 *     sticky device flag ATTN_ERR_KVLEN_RANGE (read with attn_get_device_status).
 *   - Key and value slots at or beyond kv_len[b] are never used: any content there,
 *     NaN and Inf included, leaves out and lse bit-identical.
 *   - kv_len[b] = 0 gives out = 0 and lse = -inf for every row of that element.
 *   - Supported head dims: D in {32, 64, 128, 256}.  Device: compute capability 10.0.
 */
#ifndef ATTN_PREFIX_H
#define ATTN_PREFIX_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, non-positive size, bad scale */
    ATTN_ERR_UNSUPPORTED = 2,   /* head dim not in {32,64,128,256}, or device not sm_100 */
    ATTN_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed (launch, attribute) */
    ATTN_ERR_TIMEOUT = 4,       /* a bounded in-kernel wait gave up (device flag) */
    ATTN_ERR_KVLEN_RANGE = 5    /* some kv_len[b] was outside [0, Tk] (device flag) */
} attn_status;

/* Element strides of a [B, H, T, D] operand whose d index is contiguous (stride 1):
 * element (b, h, t, d) is at base + b*b_stride + h*h_stride + t*t_stride + d.  The
 * *_strided entry points take one per operand; NULL means the contiguous [B,H,T,D]
 * layout (b = H*T*D, h = T*D, t = D).  JAX's [B, T, H, D] ("BTNH") layout is
 * {T*H*D, D, H*D}; q, k, v sliced out of one packed [B, T, 3, H, D] tensor are
 * {3*T*H*D, D, 3*H*D}.  Every stride must be a non-negative multiple of 8 elements
 * (16-byte rows, as TMA and the vector stores need) and t >= D; otherwise the call
 * returns ATTN_ERR_INVALID_ARG.  Output rows of distinct (b, h, t) must not overlap. */
typedef struct {
    int64_t b, h, t;
} attn_strides;

/* Single-pass forward.
 *   q:      bf16 [B, H, Tq, D]         k, v: bf16 [B, H, Tk, D]
 *   kv_len: int32 [B], device memory  (valid key count per batch element)
 *   out:    bf16 [B, H, Tq, D]         lse:  fp32 [B, H, Tq] natural log, or NULL
 *   scale:  finite; the usual choice is 1/sqrt(D).
 * Sizes: B, H, Tq, Tk >= 1 and B*H <= 2^31-1.  Returns ATTN_OK once the work is
 * enqueued. */
attn_status attn_prefix_fwd(const void* q, const void* k, const void* v,
                            const int32_t* kv_len, void* out, float* lse,
                            int B, int H, int Tq, int Tk, int D, float scale,
                            cudaStream_t stream);

/* attn_prefix_fwd with q, k, v and out at caller strides (see attn_strides); lse stays
 * contiguous [B, H, Tq].  Same result, bit for bit, as attn_prefix_fwd on contiguous
 * copies. */
attn_status attn_prefix_fwd_strided(const void* q, const void* k, const void* v,
                                    const int32_t* kv_len, void* out, float* lse,
                                    int B, int H, int Tq, int Tk, int D, float scale,
                                    const attn_strides* q_strides, const attn_strides* k_strides,
                                    const attn_strides* v_strides, const attn_strides* out_strides,
                                    cudaStream_t stream);

/* Keys per split chunk for a given key buffer length and split count: ceil(Tk/C)
 * rounded up to the 128-key tile.  Chunk c covers keys [c*L, min((c+1)*L, kv_len[b])).
 * Returns 0 for invalid arguments. */
int attn_split_chunk_len(int Tk, int num_splits);

/* Bytes of one contiguous workspace holding part_out followed by part_lse at a
 * 256-byte aligned offset (attn_split_lse_offset): the caller may carve both from it. */
size_t attn_split_workspace_bytes(int num_splits, int B, int H, int Tq, int D);
size_t attn_split_lse_offset(int num_splits, int B, int H, int Tq, int D);

/* Split-KV partial forward: for every chunk c < num_splits, the attention of each query
 * row over the keys of that chunk alone, normalised, plus its log-sum-exp.  A chunk
 * holding no valid key yields part_out = 0 and part_lse = -inf.
 *   part_out: fp32 [num_splits, B, H, Tq, D]     part_lse: fp32 [num_splits, B, H, Tq]
 * num_splits in [1, 1024].  Other arguments as attn_prefix_fwd. */
attn_status attn_prefix_fwd_split(const void* q, const void* k, const void* v,
                                  const int32_t* kv_len, int num_splits,
                                  float* part_out, float* part_lse,
                                  int B, int H, int Tq, int Tk, int D, float scale,
                                  cudaStream_t stream);

/* attn_prefix_fwd_split with q, k, v at caller strides; the partials keep the layout
 * above. */
attn_status attn_prefix_fwd_split_strided(const void* q, const void* k, const void* v,
                                          const int32_t* kv_len, int num_splits,
                                          float* part_out, float* part_lse,
                                          int B, int H, int Tq, int Tk, int D, float scale,
                                          const attn_strides* q_strides, const attn_strides* k_strides,
                                          const attn_strides* v_strides, cudaStream_t stream);

/* Exact log-sum-exp combination of split partials (same layouts as above):
 *   M = max_c lse_c;  lse = M + ln sum_c exp(lse_c - M);  out = sum_c exp(lse_c - lse) O_c
 * Rows whose every partial is empty give out = 0, lse = -inf.
 *   out: bf16 [B, H, Tq, D]    lse: fp32 [B, H, Tq] or NULL */
attn_status attn_lse_combine(const float* part_out, const float* part_lse, int num_splits,
                             void* out, float* lse, int B, int H, int Tq, int D,
                             cudaStream_t stream);
/* attn_lse_combine writing out at caller strides (lse stays contiguous). */
attn_status attn_lse_combine_strided(const float* part_out, const float* part_lse, int num_splits,
                                     void* out, float* lse, int B, int H, int Tq, int D,
                                     const attn_strides* out_strides, cudaStream_t stream);

/* Split-KV forward with the combine fused into the same launch: the split partials of
 * attn_prefix_fwd_split, then, inside the kernel, the exact combination of
 * attn_lse_combine.  The pages combine shard results by log-sum-exp weights so that
 * only softmax statistics cross ("Add sequence-parallel multi-GPU inference ...",
 * section "Sequence-parallel inference"); here the last chunk to finish a 128-row
 * query tile combines that tile, so no second launch re-reads the partials from DRAM.
 *   workspace: device memory of attn_split_fused_workspace_bytes(num_splits, B, H, Tq, D)
 *     bytes, 16-byte aligned, owned by the caller: part_out at offset 0, part_lse at
 *     attn_split_lse_offset, then B*H*ceil(Tq/128) int32 tile counters at
 *     attn_split_counter_offset.  The counters must be zero before the first call
 *     (e.g. one cudaMemsetAsync of the workspace); every call that completes leaves them
 *     zero again, so a workspace is reused without clearing.  After a call that raised
 *     a device error flag (attn_get_device_status != ATTN_OK), zero them again.  Calls
 *     sharing one workspace must not overlap on the GPU.
 *   out: bf16 [B,H,Tq,D]; lse: fp32 [B,H,Tq] or NULL.  Same result, bit for bit, as
 *   attn_prefix_fwd_split followed by attn_lse_combine.  Other arguments and checks as
 *   attn_prefix_fwd_split. */
size_t attn_split_counter_offset(int num_splits, int B, int H, int Tq, int D);
size_t attn_split_fused_workspace_bytes(int num_splits, int B, int H, int Tq, int D);
attn_status attn_prefix_fwd_split_fused(const void* q, const void* k, const void* v,
                                        const int32_t* kv_len, int num_splits, void* workspace,
                                        void* out, float* lse,
                                        int B, int H, int Tq, int Tk, int D, float scale,
                                        cudaStream_t stream);

/* Multi-range key mask: batch element b attends to the keys of its num_segments (S)
 * segments instead of one prefix,
 *     [seg_start[b*S + s], seg_start[b*S + s] + seg_len[b*S + s]),   s = 0 .. S-1,
 * taken together.  This is the gathered-shards K/V of "Add sequence-parallel multi-GPU
 * inference ..." (section "Sequence-parallel inference"): every device's context K/V
 * is gathered with padded key slots, so the valid keys are one range per shard.
 *   seg_start, seg_len: int32 [B, S], DEVICE memory; the host never reads them.
 *   S in [1, 4096].  A segment is intersected with [0, Tk); a negative length counts
 *   as 0; a key in two segments takes part twice; the keys of all segments are cut
 *   after Tk keys.  A negative length, a non-empty segment reaching outside [0, Tk) or a
 *   cut raises the sticky ATTN_ERR_KVLEN_RANGE flag.  Slots outside every segment are
 *   never read: any content there leaves out and lse bit-identical.  An element with no
 *   valid key gives out = 0, lse = -inf.
 *   workspace: attn_segments_workspace_bytes(B, H, Tk, D) bytes of device memory,
 *   16-byte aligned, owned by the caller (no initialisation needed).  One kernel
 *   gathers the segments' K and V rows into it as a contiguous prefix per element;
 *   the prefix kernel then runs on the gathered rows (so the result equals
 *   attn_prefix_fwd on those rows, bit for bit).
 *   Other arguments and checks as attn_prefix_fwd. */
size_t attn_segments_workspace_bytes(int B, int H, int Tk, int D);
attn_status attn_prefix_fwd_segments(const void* q, const void* k, const void* v,
                                     const int32_t* seg_start, const int32_t* seg_len,
                                     int num_segments, void* workspace, void* out, float* lse,
                                     int B, int H, int Tq, int Tk, int D, float scale,
                                     cudaStream_t stream);

/* Split-KV forward that allocates nothing, for callers that cannot call cudaMalloc.
 * The pages have no counterpart to this entry point: it exists for the integration
 * side, not for the method.  Some callers only ever receive device memory for their
 * inputs and outputs: a hook running inside another framework whose allocator owns all
 * of device memory, a runtime that fixes its memory plan at start-up, or a real-time
 * loop that cannot take the device-wide synchronisation a cudaMalloc may imply.  For
 * them the split partials live in one file-scope device array of the library
 * (ATTN_NOALLOC_SCRATCH_BYTES = 64 MiB), which every GPU that loads the library holds
 * until the process exits.
 *   Same arguments and result as attn_prefix_fwd_split followed by attn_lse_combine:
 *   out bf16 [B,H,Tq,D], lse fp32 [B,H,Tq] or NULL.
 *   Shapes whose split workspace, attn_split_workspace_bytes(num_splits, B, H, Tq, D),
 *   exceeds ATTN_NOALLOC_SCRATCH_BYTES are rejected with ATTN_ERR_INVALID_ARG before any
 *   CUDA call.
 *   The first call on a device looks up the array's device address (with that device
 *   current); make that first call before any stream capture.  After a device reset
 *   (a new context on the device) the next call looks the address up again.
 *   Every call shares the one array and leaves its partials there; each call writes
 *   every partial it reads, so nothing needs clearing, but calls whose work overlaps on
 *   the GPU (other streams, other host threads) race on the array and must be serialised
 *   by the caller. */
#define ATTN_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
attn_status attn_prefix_fwd_splitkv_noalloc(const void* q, const void* k, const void* v,
                                            const int32_t* kv_len, int num_splits,
                                            void* out, float* lse,
                                            int B, int H, int Tq, int Tk, int D, float scale,
                                            cudaStream_t stream);

/* Synchronizes `stream`, then reads and clears the sticky device flags raised by
 * earlier launches: ATTN_ERR_TIMEOUT has priority over ATTN_ERR_KVLEN_RANGE; ATTN_OK if
 * none.  A CUDA error during the synchronization returns ATTN_ERR_CUDA. */
attn_status attn_get_device_status(cudaStream_t stream);

/* Upper bound, in nanoseconds, on every in-kernel wait (default 1e9 = 1 s).  A wait that
 * runs out makes its CTA stop, drain its copies in flight, free its tensor memory and
 * exit, and raises ATTN_ERR_TIMEOUT.  Values below 1e6 are raised to 1e6. */
void attn_set_wait_limit_ns(uint64_t ns);

/* Test hooks, for tests only.  They are process-wide settings (atomics) that apply to
 * every launch, from any host thread, started after the call.
 * ATTN_DEBUG_DROP_COPY makes the copy producer of the next launches
 * announce one key-tile copy without issuing it, so that the consumer's bounded wait
 * runs out (exercises the ATTN_ERR_TIMEOUT path without faulting anything).  0 = off. */
#define ATTN_DEBUG_DROP_COPY 1u
/* Test hook: run head dims 128 and 256 on the single-CTA kernel instead of the CTA-pair
 * kernel (for side-by-side checks of the two implementations). */
#define ATTN_DEBUG_SINGLE_CTA 2u
void attn_set_debug_flags(unsigned flags);

/* Human-readable name of a status code (static string). */
const char* attn_status_string(attn_status s);

/* Library version, major*10000 + minor*100 + patch. */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_PREFIX_H */
