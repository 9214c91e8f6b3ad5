/*
 * fa.h -- C ABI of the B200 (sm_100a) fused exact-attention kernels: the
 * forward pass (fa_fwd and its variants for different query/key lengths,
 * split keys, variable-length batches and 8-bit inputs) and the backward
 * pass (fa_bwd).  The common definitions follow; each variant states what it
 * adds or changes at its declaration.
 *
 * The operation
 * -------------
 * For every batch index b and head h, with query rows i and key rows j of
 * one sequence of length N and head dimension d:
 *
 *     S_ij  = scale * sum_t Q[b,h,i,t] * K[b,h,j,t]
 *     O_i   = sum_{j in vis(i)} softmax_j(S_i.) * V[b,h,j,:]
 *     lse_i = ln sum_{j in vis(i)} exp(S_ij)
 *
 * This is scaled dot-product attention as stated in "理解 Flash Attention：在
 * Triton 中从头编写算法" (section "什么是注意力"), computed exactly (wmrh.cn
 * FlashAttention article, introduction: no accuracy is traded for speed) in
 * one pass with the online softmax of AllenY's blog "FlashAttention" post
 * (sections "从3-pass到2-pass" and "FlashAttention"): the N x N score matrix is
 * never written to memory.  lse is the natural-log logsumexp of the scaled
 * scores of each row (kept so a backward pass can recompute S).
 *
 * Visibility vis(i): every key; intersected with {j <= i} when `causal` is 1;
 * intersected with {j : block_mask[b,h,i/128,j/128] != 0} when `block_mask`
 * is non-NULL (block-sparse attention: a masked 128 x 128 block contributes
 * nothing and is never loaded or multiplied).  A row whose vis(i) is empty
 * gets O_i = 0 and lse_i = -inf.
 *
 * Layouts and types (all buffers are owned by the caller; the library
 * allocates nothing per call and keeps no pointer after the call returns):
 *   q, k, v, o   device memory, bfloat16, contiguous [B, H, N, d] (d fastest),
 *                16-byte aligned.
 *   lse          device memory, float32, contiguous [B, H, N], 4-byte aligned.
 *                No byte of o or lse may lie inside q, k, v, block_mask or
 *                the other output (checked by address range; inputs may
 *                overlap each other).
 *   block_mask   NULL, or device memory, uint8, contiguous
 *                [B, H, ceil(N/128), ceil(N/128)], 1 (non-zero) = keep.
 *   d            64 or 128.
 *   scale        finite and > 0 (usually 1/sqrt(d)).
 *   causal       0 or 1.
 *   N            any value >= 1; a ragged last tile is masked inside the kernel.
 *
 * Errors: every entry point returns an fa_status.  Argument errors are found
 * before anything is launched.  Launches are asynchronous: a fault inside the
 * kernel surfaces at the caller's next synchronisation; a device-side wait
 * that exceeded its time limit is reported by fa_device_status().  No C++
 * exception crosses this interface.  The entry points may be called from
 * several host threads; per-device set-up is done once, under a lock, by the
 * first call of any entry point on that device (it loads the library's
 * device code, whose fixed arrays are then reserved; see
 * fa_fwd_splitkv_noalloc).
 */
#ifndef FA_B200_FA_H_
#define FA_B200_FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FA_MASK_BLOCK 128

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

typedef enum fa_status {
  FA_OK = 0,
  FA_ERR_INVALID_ARGUMENT = 1, /* null/misaligned/host pointer, bad size, scale, causal */
  FA_ERR_UNSUPPORTED = 2,      /* d not in {64,128}, not an sm_100 device, size limits */
  FA_ERR_CUDA = 3,             /* a CUDA runtime/driver call failed: see fa_last_cuda_error() */
  FA_ERR_DEVICE_TIMEOUT = 4    /* a device-side wait gave up (reported by fa_device_status) */
} fa_status;

/*
 * Fused attention forward on the legacy default stream (stream 0).
 * Writes o [B,H,N,d] and lse [B,H,N]; see the header comment for meaning.
 */
FA_API int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
           int d, float scale, int causal, const uint8_t* block_mask);

/*
 * The same, enqueued on `cuda_stream` (a cudaStream_t; NULL = legacy default
 * stream).  The call returns once the kernel is enqueued.
 */
FA_API int fa_fwd_stream(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                  int N, int d, float scale, int causal, const uint8_t* block_mask,
                  void* cuda_stream);

/*
 * The forward pass of fa_fwd_stream for inputs and outputs in host memory,
 * with the host<->device transfers overlapped with the computation.
 *
 * q_host, k_host, v_host (bf16 [B,H,N,d]), o_host (bf16 [B,H,N,d]) and
 * lse_host (fp32 [B,H,N]) are host memory owned by the caller; page-locked
 * memory lets the copies overlap each other and the kernels (pageable memory
 * works, but its copies do not overlap).  q_dev ... lse_dev are device
 * buffers of the same sizes, owned by the caller, through which the data
 * pass (afterwards they hold the inputs and the results as well).
 * block_mask: NULL or device memory, as for fa_fwd.
 *
 * The B*H heads are taken in up to 16 chunks of whole heads.  Chunk c's Q, K
 * and V are copied in on an internal stream while the chunks before it are
 * computed on cuda_stream and their O and lse are copied out on a second
 * internal stream (a copy engine per direction).  Each chunk is computed by
 * the same kernel as fa_fwd_stream, so the results are bit for bit those of
 * fa_fwd_stream.  Ordering: the call's work starts after the work enqueued on
 * cuda_stream before it, and everything it does, the copies into o_host and
 * lse_host included, is complete once cuda_stream has passed the point of
 * the call's return: synchronise cuda_stream before reading o_host.  The
 * host buffers must stay valid until then.  The internal streams and events
 * are created on the first call on each device and kept; calls on one device
 * share them, so the copies of concurrent calls run one call after another.
 *
 * Returns FA_OK, FA_ERR_INVALID_ARGUMENT (a null pointer, a *_dev pointer
 * that is not device memory or a *_host pointer that is, sizes, scale or
 * causal as for fa_fwd, o_dev / lse_dev overlapping an input buffer, o_host /
 * lse_host overlapping q_host, k_host, v_host or each other),
 * FA_ERR_UNSUPPORTED or FA_ERR_CUDA.
 */
FA_API int fa_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                       float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                       float* lse_dev, int B, int H, int N, int d, float scale, int causal,
                       const uint8_t* block_mask, void* cuda_stream);

/*
 * Attention with Nq query rows and Nk keys per (b, h) -- cross-attention, or
 * decoding against a key/value cache.  q, o: [B, H, Nq, d]; k, v: [B, H, Nk, d];
 * lse: [B, H, Nq]; block_mask: NULL or [B, H, ceil(Nq/128), ceil(Nk/128)].
 * With `causal`, key j is visible to query i iff j <= i + (Nk - Nq): the
 * queries are the last Nq positions of the sequence (the diagonal is aligned
 * to the last key; for Nq = Nk this is j <= i).  When Nq > Nk the first
 * Nq - Nk rows see no key and get O = 0, lse = -inf.  Otherwise identical to
 * fa_fwd_stream; fa_fwd_stream(..., N, ...) equals fa_fwd_qk(..., N, N, ...).
 * The problem statement this generalises is the one of fa_fwd (scaled
 * dot-product attention, "理解 Flash Attention" section "什么是注意力");
 * different lengths and the causal alignment are this library's extension.
 */
FA_API int fa_fwd_qk(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int Nq, int Nk, int d, float scale, int causal,
                     const uint8_t* block_mask, void* cuda_stream);

/*
 * Split-key ("flash-decoding") forward for problems with fewer work units than
 * SMs, such as decoding against a long key/value cache.  The keys are cut into
 * `num_splits` slices of whole 128-key tiles (at most 256; slices that would be
 * empty are dropped).  Each work unit computes one slice's normalised partial
 * output and logsumexp into `workspace`.  A second kernel merges the slices
 * with the concatenated-softmax rule ("理解 Flash Attention", section
 * "瓦片注意力计算") into o and lse.  Arguments and meaning are those of
 * fa_fwd_qk.  The results equal fa_fwd_qk's up to floating-point rounding
 * (they are not bitwise identical).
 * workspace: device memory, 16-byte aligned, at least
 *   fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, num_splits) bytes, owned by
 *   the caller and overwritten by the call.  It may be NULL when that size is 0
 *   (a single slice); otherwise its first that many bytes may not overlap any
 *   other buffer of the call.
 * Calls that share one workspace must not overlap on the GPU.  Two launches are
 * enqueued on `cuda_stream` when there is more than one slice.
 */
FA_API int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int H, int Nq, int Nk, int d, float scale, int causal,
                          const uint8_t* block_mask, int num_splits, void* workspace,
                          size_t workspace_bytes, void* cuda_stream);

/* Workspace bytes fa_fwd_splitkv needs (0 when it uses a single slice). */
FA_API size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d, int num_splits);

/* Size of the fixed device array behind fa_fwd_splitkv_noalloc (16 MiB). */
#define FA_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * fa_fwd_splitkv without a caller workspace, for callers that cannot allocate
 * device memory at call time.  Examples: plugin code run by a host framework
 * that owns every allocation; code on a latency-critical path that may not pay
 * for cudaMalloc; code that runs while allocation is forbidden.  The partial
 * results live in one fixed array of FA_NOALLOC_SCRATCH_BYTES in the library's
 * device memory.  Every GPU that loads the library holds it until the process
 * exits.  The call itself allocates nothing: it makes no cudaMalloc or
 * cudaFree call, and no call to any allocating library.
 *
 * Arguments and results are those of fa_fwd_splitkv (num_splits >= 1), minus
 * the workspace.  A problem whose workspace would exceed the array
 * (fa_fwd_splitkv_workspace_bytes(...) > FA_NOALLOC_SCRATCH_BYTES) is rejected
 * with FA_ERR_UNSUPPORTED before anything is launched.
 *
 * The array is reserved when the library's device code is loaded, which the
 * first call of any entry point on a device does, together with the set-up
 * that looks up the array's device address (cudaGetSymbolAddress, once per
 * device, with that device current).  A caller that may not allocate at call
 * time makes one call at initialisation (fa_device_status is enough), and
 * that first call comes before any stream capture.  Argument errors are
 * found before any CUDA call, as for the other entry points.
 *
 * All calls on a device share the one array, and it keeps the last call's
 * contents.  Calls whose kernels overlap on the GPU (on different streams,
 * without ordering between them) race on it and corrupt each other's results:
 * serialise them.  No part of the array needs to start at zero.  After a
 * call whose kernel gave up on a wait (fa_device_status reports
 * FA_ERR_DEVICE_TIMEOUT), its o and lse are undefined and may hold values
 * merged from an earlier call's partial results.
 *
 * The pages have no counterpart to this entry point: it is a packaging of
 * fa_fwd_splitkv for callers without an allocator.
 */
FA_API int fa_fwd_splitkv_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                  int B, int H, int Nq, int Nk, int d, float scale, int causal,
                                  const uint8_t* block_mask, int num_splits, void* cuda_stream);

/*
 * A slice count that keeps all SMs of the current device busy: 1 when the
 * problem already has at least one work unit per SM, otherwise about two
 * waves of units, each slice at least two key tiles long.
 */
FA_API int fa_fwd_splitkv_heuristic(int B, int H, int Nq, int Nk);

/*
 * 8-bit forward: the same attention on FP8 (e4m3) inputs, the low-precision
 * direction the pages name for the next FlashAttention generation
 * (wmrh.cn article, section "FlashAttention 的局限和后续发展").  q, k, v hold
 * e4m3 codes (OCP FP8 E4M3: bias 7, no infinities, largest finite 448)
 * standing for q_descale * q, k_descale * k, v_descale * v; the result is the
 * attention of those real values, exactly as fa_fwd_qk defines it:
 *   O = softmax(scale * (q_descale q)(k_descale k)^T) (v_descale v).
 * Both products run on the 8-bit tensor-core path (kind::f8f6f4) with fp32
 * accumulation; P is rounded to e4m3 before the PV product and the row sums
 * add those same rounded values, so every O row is an exact weighted mean of
 * V rows with each weight off by at most 2^-4 relative.
 *
 * q: [B, H, Nq, d]; k, v: [B, H, Nk, d], one byte per element, contiguous,
 * 16-byte aligned; o: bf16 [B, H, Nq, d]; lse: fp32 [B, H, Nq] (natural log
 * of the scaled scores, as fa_fwd).  d must be 128.  causal and block_mask as
 * in fa_fwd_qk.  Descales finite and > 0.  Asynchronous on cuda_stream.
 *
 * Returns FA_OK, FA_ERR_INVALID_ARGUMENT (as fa_fwd_qk, or a bad descale),
 * FA_ERR_UNSUPPORTED (d != 128, sizes as fa_fwd_qk) or FA_ERR_CUDA.
 */
FA_API int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int Nq, int Nk, int d, float scale, int causal,
                      const uint8_t* block_mask, float q_descale, float k_descale,
                      float v_descale, void* cuda_stream);

/*
 * Variable-length batch: B independent attention problems of different
 * lengths in one launch, the layout of packed token streams.  Sequence b
 * owns query token rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key/value
 * rows [cu_seqlens_k[b], cu_seqlens_k[b+1]); its queries attend to its own
 * keys only, each sequence computed exactly as fa_fwd_qk computes one head
 * (same softmax, same bottom-right causal rule j <= i + (nk_b - nq_b), an
 * empty sequence or a query row with no visible key gives O = 0,
 * lse = -inf).  The pages treat one sequence; batching unequal lengths
 * without padding is this library's extension of the same loop.
 *
 * q, o: bf16 [total_q, H, d]; k, v: bf16 [total_k, H, d] (token-major, d
 * fastest); lse: fp32 [H, total_q].  cu_seqlens_q / cu_seqlens_k: int32
 * device arrays of B+1 non-decreasing offsets starting at 0 and ending at
 * total_q / total_k.  max_seqlen_q, the longest query length, sizes the
 * launch only: the work of each sequence follows its own offsets, read on
 * the device.  Batches of more than 4096 sequences take one launch per 4096
 * on cuda_stream.  Offsets outside [0, total] are clamped on the device
 * (so no access leaves the buffers), but such a batch has no defined result.
 * No block mask.  All pointers device memory owned by the caller, 16-byte
 * aligned (lse, cu_seqlens: 4).  Asynchronous on cuda_stream.
 *
 * Returns FA_OK, FA_ERR_INVALID_ARGUMENT (null, host or misaligned pointer,
 * B, H, total_q, total_k or max_seqlen_q < 1, bad scale or causal, o
 * or lse overlapping an input or each other), FA_ERR_UNSUPPORTED (d not 64 or 128, no sm_100
 * device, more than 2^31 work units or query rows x H) or FA_ERR_CUDA.
 */
FA_API int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                         const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H,
                         int total_q, int total_k, int max_seqlen_q, int d, float scale,
                         int causal, void* cuda_stream);

/*
 * Backward pass: dQ, dK, dV of the forward above for the upstream gradient
 * dO.  The scores are recomputed from q, k and the forward's lse, not stored
 * ("理解 Flash Attention", section "瓦片注意力计算"), with P = exp(S - lse),
 *   dV = P^T dO,  dP = dO V^T,  D_i = dO_i . O_i,  dS = P o (dP - D),
 *   dQ = scale dS K,  dK = scale dS^T Q.
 * q, o, dout, dq: bf16 [B, H, Nq, d]; k, v, dk, dv: bf16 [B, H, Nk, d]; lse:
 * fp32 [B, H, Nq] as written by the forward; causal, block_mask, scale and d
 * exactly as passed to the forward (fa_fwd / fa_fwd_qk).  All device memory,
 * 16-byte aligned (lse: 4), owned by the caller; no byte of dq, dk, dv or
 * the workspace may lie inside an input or another of them (checked by
 * address range).
 * workspace: device memory of at least fa_bwd_workspace_bytes(B, H, Nq) bytes,
 *   16-byte aligned, overwritten (it receives D).  Calls sharing a workspace
 *   must not overlap on the GPU.
 * Two kernels are enqueued on `cuda_stream` (dQ with D, then dK and dV).
 */
FA_API int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* dout, void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk,
                  int d, float scale, int causal, const uint8_t* block_mask, void* workspace,
                  size_t workspace_bytes, void* cuda_stream);

/* Workspace bytes fa_bwd needs: one fp32 per query row, rounded to 16. */
FA_API size_t fa_bwd_workspace_bytes(int B, int H, int Nq);

/*
 * Reads and clears the device-side status word of the current device after
 * synchronising `cuda_stream`.  Returns FA_OK, FA_ERR_DEVICE_TIMEOUT (a
 * kernel's wait on one of its own barriers exceeded the time limit; the
 * kernel then stopped early and released its resources, and its outputs
 * are undefined) or FA_ERR_CUDA.
 */
FA_API int fa_device_status(void* cuda_stream);

/* Human-readable name of a status code (static storage, never NULL). */
FA_API const char* fa_status_string(int status);

/* The cudaError_t value behind the last FA_ERR_CUDA on this host thread. */
FA_API int fa_last_cuda_error(void);

/* Number of kernel launches one fa_fwd / fa_fwd_qk / fa_fwd_fp8 call makes
 * (constant: 1).  fa_fwd_varlen makes one per 4096 sequences, fa_fwd_host one
 * per chunk of heads, fa_fwd_splitkv with more than one slice 2 (the forward
 * and the merge), fa_bwd 2 (the dQ and the dK/dV launches). */
FA_API int fa_launches_per_call(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_H_ */
