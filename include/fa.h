/*
 * fa.h -- C ABI of the B200 (sm_100a) exact attention forward library
 *         (libfa.so).
 *
 * The operation: O = softmax(scale * Q K^T + mask) V for every (batch, head),
 * computed tile by tile with the online softmax, never writing the L_q x L_k
 * score matrix to memory, plus the per-row log-sum-exp of the scaled, masked
 * scores.
 *   - formulas: "PyTorch Transformer Flash Attention机制" section 1;
 *     "FlashAttention算法原理与性能优化实战" section 1.1;
 *   - online softmax: "Flash Attention是怎么做到又快又省显存的？" (Online
 *     normalizer derivation) and "FlashAttention算法原理与性能优化实战"
 *     section 1.2.2;
 *   - operator statement (4-D [B,H,S,D] inputs, output shaped like the query,
 *     fp32 softmax statistics of shape [B,H,S], scale_value, pre_tokens /
 *     next_tokens window): "FlashAttention算法原理与性能优化实战" section 2.2;
 *   - logsumexp kept for the backward pass: Triton FA2 walkthrough;
 *   - MQA/GQA and the causal mask: "FlashAttention算法原理与性能优化实战"
 *     section 1.3.
 *
 * All functions return 0 (FA_OK) or a negative fa_status; none aborts.
 * Every pointer argument marked "device" must point to memory the current
 * CUDA device can read/write; the library allocates no memory and keeps no
 * state between calls other than one device-side status word and the
 * static scratch of fa_fwd_splitkv_static (module memory, not allocated by
 * any call).
 */
#ifndef FA_H
#define FA_H

#include <stddef.h>
#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_F16 = 0,  /* IEEE binary16 */
    FA_BF16 = 1  /* bfloat16 */
} fa_dtype;

typedef enum {
    FA_MASK_NONE = 0,
    FA_MASK_BOOL = 1,   /* uint8; nonzero hides the key */
    FA_MASK_F16 = 2,    /* IEEE binary16, added to the scaled score */
    FA_MASK_F32 = 3     /* binary32, added to the scaled score */
} fa_mask_type;

typedef enum {
    FA_OK = 0,
    FA_ERR_NULL = -1,     /* q or out is NULL while L_q > 0, or k or v is
                             NULL while L_k > 0 */
    FA_ERR_SHAPE = -2,    /* B, H, H_kv < 1; L_q, L_k < 0; H % H_kv != 0;
                             or a size whose byte extent overflows */
    FA_ERR_HEADDIM = -3,  /* D not supported: the 16-bit forward entries take
                             any multiple of 16 in [16, 128]; fa_fwd_fp8
                             takes 32, 64, 128 */
    FA_ERR_DTYPE = -4,    /* dtype not FA_F16 / FA_BF16 */
    FA_ERR_ALIGN = -5,    /* q, k, v, out not 16-byte aligned, or lse not
                             4-byte aligned */
    FA_ERR_ARG = -6,      /* scale is negative, NaN or infinite */
    FA_ERR_CUDA = -7,     /* a CUDA runtime/driver call failed (launch,
                             tensor-map encoding, device query) */
    FA_ERR_TIMEOUT = -8,  /* a device-side wait gave up (watchdog); the
                             outputs of that launch are not valid */
    FA_ERR_WORKSPACE = -9, /* workspace smaller than the size the matching
                              *_workspace_bytes() call returns */
    FA_ERR_SCRATCH = -10   /* fa_fwd_splitkv_static: the problem needs more
                              than FA_STATIC_SCRATCH_BYTES of scratch */
} fa_status;

/*
 * fa_fwd -- exact attention forward on `stream` (asynchronous).
 *
 *   q     device, [B, H,    L_q, D] contiguous, element type `dtype`
 *   k, v  device, [B, H_kv, L_k, D] contiguous, element type `dtype`
 *   out   device, [B, H,    L_q, D] contiguous, element type `dtype`
 *         (written; RNE rounding of the fp32 result)
 *   lse   device, [B, H, L_q] contiguous fp32, or NULL to skip it.
 *         lse = ln(sum_j exp(scale * q_i . k_j)) over the visible keys j;
 *         -inf for a row with no visible key (whose out row is 0).
 *   scale finite, >= 0 (the pages use 1/sqrt(D); this ABI has no default).
 *   causal, window_left, window_right:
 *         key j is visible from query i iff j < L_k and
 *         (window_left  < 0 or j >= i - window_left) and
 *         (window_right < 0 or j <= i + window_right) and
 *         (causal == 0 or j <= i).  Indices are raw positions (row i of Q
 *         and row j of K), so causal == 1 equals window_right = 0.
 *         A negative window means unbounded (the pages' INT_MAX default).
 *   GQA / MQA: query head h reads key/value head h / (H / H_kv).
 *   L_q == 0 is a no-op; L_k == 0 writes out = 0 and lse = -inf.  A
 *   pointer to a tensor with no elements may be NULL.
 *
 * Buffers are owned by the caller and must not overlap out/lse with inputs.
 * The call only enqueues work: argument errors are returned before anything
 * is enqueued; device-side watchdog errors are reported by
 * fa_get_device_status().
 *
 * Decoding shapes -- at most two query rows per K/V head (L_q * H / H_kv
 * <= 2) and D in {16, 32, 64, 128} -- run on a CUDA-core kernel that
 * streams the key/value cache through shared memory (the product with one
 * or two query rows is a matrix-vector product, far from the tensor cores'
 * work); it keeps the softmax weights in fp32.  Everything else runs on the
 * tcgen05 tensor-core kernel.  The result is the same function either way.
 */
int fa_fwd(const void *q, const void *k, const void *v, void *out, float *lse,
           int B, int H, int H_kv, int L_q, int L_k, int D, float scale,
           int causal, int window_left, int window_right, int dtype,
           cudaStream_t stream);

/*
 * fa_fwd_ex -- fa_fwd with the optional inputs and outputs of the operator
 * statement in "FlashAttention算法原理与性能优化实战" §2.2: an attention mask
 * and the two softmax statistics kept for the backward pass.
 *
 *   mask, mask_type  device, or NULL with FA_MASK_NONE.  Element
 *               (b, h, i, j) is mask[b*mask_stride_b + h*mask_stride_h +
 *               i*mask_stride_q + j] (strides in elements, >= 0; a stride
 *               of 0 broadcasts, e.g. [L_q, L_k] for every batch and head:
 *               0, 0, L_k).  FA_MASK_BOOL: a nonzero byte hides key j from
 *               query i.  FA_MASK_F16 / FA_MASK_F32: the value is added to
 *               scale * q_i . k_j before the softmax (-inf hides).  The
 *               causal / window rule applies on top.  The caller guarantees
 *               every addressed element lies in the buffer.  16-byte
 *               aligned base and strides take the vectorised load path.
 *   softmax_max, softmax_sum  device [B, H, L_q] fp32, both or neither
 *               (NULL): the row max m_i of the scaled, masked scores and
 *               sum_j exp(s_ij - m_i); lse = m + ln(sum).  A row with no
 *               visible key gets -inf and 0.
 * Other arguments, errors and edge cases as fa_fwd; FA_ERR_ARG for a bad
 * mask_type or a negative stride.
 */
int fa_fwd_ex(const void *q, const void *k, const void *v, void *out, float *lse,
              float *softmax_max, float *softmax_sum, const void *mask, int mask_type,
              long long mask_stride_b, long long mask_stride_h, long long mask_stride_q,
              int B, int H, int H_kv, int L_q, int L_k, int D, float scale, int causal,
              int window_left, int window_right, int dtype, cudaStream_t stream);

/*
 * fa_fwd_fp8 -- exact attention forward on fp8 (E4M3) inputs.  The pages
 * list fp8 among FlashAttention-2's input types ("PyTorch Transformer Flash
 * Attention机制" §5) without details; this entry reads them as: q, k, v hold
 * E4M3 codes (OCP "fn" encoding: bias 7, no infinities, largest 448) whose
 * real values are code * descale_{q,k,v}; the scores are
 * scale * descale_q * descale_k * (q_i . k_j) accumulated in fp32; P enters
 * the P.V product rounded to E4M3 (the tensor cores' fp8 kind takes both
 * operands in 8 bits) while the normaliser sums the unrounded fp32 weights;
 * O = descale_v * P.V / l is written as bf16.
 *
 *   q         device, [B, H,    L_q, D] E4M3 codes (1 byte each)
 *   k, v      device, [B, H_kv, L_k, D] E4M3 codes
 *   out       device, [B, H,    L_q, D] bfloat16 (written)
 *   lse       device, [B, H, L_q] fp32 or NULL (natural log, as fa_fwd)
 *   descale_q, descale_k, descale_v  finite, >= 0 (1 = codes are the values)
 *   D in {32, 64, 128} (rows of at least 32 bytes), else FA_ERR_HEADDIM.
 * Masks, windows, GQA, edge cases and errors as fa_fwd.
 */
int fa_fwd_fp8(const void *q, const void *k, const void *v, void *out, float *lse, int B,
               int H, int H_kv, int L_q, int L_k, int D, float scale, float descale_q,
               float descale_k, float descale_v, int causal, int window_left,
               int window_right, cudaStream_t stream);

/*
 * fa_fwd_host_workspace_bytes -- bytes of device workspace fa_fwd_host
 * needs (0 if the sizes are invalid): two slots, each holding one chunk's
 * q, k, v, out and lse.
 */
size_t fa_fwd_host_workspace_bytes(int B, int H, int H_kv, int L_q, int L_k, int D,
                                   int n_chunks);

/*
 * fa_fwd_host -- fa_fwd on HOST buffers (pinned memory lets the copies run
 * asynchronously and overlap; pageable memory works but serialises them).
 * The B*H_kv key/value heads (with their query heads) are cut into
 * n_chunks contiguous ranges; chunk c's q, k, v are copied in on a copy
 * stream, its forward runs on `stream`, its out and lse are copied back on
 * a second copy stream, each chunk through one of two device slots in
 * `workspace`, so the copies in both directions overlap the kernels of
 * neighbouring chunks.  Arguments as fa_fwd except:
 *   q, k, v, out, lse  HOST pointers, same layouts (lse may be NULL)
 *   workspace          device, 256-byte aligned, at least
 *                      fa_fwd_host_workspace_bytes(...) bytes
 *   n_chunks           >= 1 (FA_ERR_ARG otherwise)
 * Returns after enqueueing; `stream` is ordered after the last copy out, so
 * synchronising it makes out and lse valid.  The copy streams and events
 * are created by the first call on each device (make it before any stream
 * capture); calls on one device must not overlap.
 */
int fa_fwd_host(const void *q, const void *k, const void *v, void *out, float *lse, int B,
                int H, int H_kv, int L_q, int L_k, int D, float scale, int causal,
                int window_left, int window_right, int dtype, void *workspace,
                size_t workspace_bytes, int n_chunks, cudaStream_t stream);

/*
 * fa_splitkv_workspace_bytes -- bytes of device workspace fa_fwd_splitkv
 * needs for these sizes (0 if the sizes are invalid): B*H*L_q*n_splits rows
 * of a D-wide fp32 partial output plus an (m, l) pair each.
 */
size_t fa_splitkv_workspace_bytes(int B, int H, int L_q, int D, int n_splits);

/*
 * fa_fwd_splitkv -- the same forward as fa_fwd, computed in n_splits
 * (1..64) slices of each query tile's key range: one launch writes every
 * slice's unnormalised output and (running max, normaliser) to `workspace`,
 * a second launch merges the slices of each row with the online-softmax
 * rescaling ("FlashAttention算法原理与性能优化实战" §1.2.2).  Meant for
 * shapes with few query tiles and long key ranges (decoding), where fa_fwd
 * would leave most SMs idle.  Arguments as fa_fwd, plus
 *   n_splits         number of key slices, 1..64 (FA_ERR_ARG otherwise)
 *   workspace        device, 256-byte aligned, caller-owned, at least
 *                    fa_splitkv_workspace_bytes(B, H, L_q, D, n_splits)
 *                    bytes (FA_ERR_WORKSPACE if smaller, FA_ERR_NULL if
 *                    NULL while L_q, L_k > 0); its contents on entry do not
 *                    matter and are overwritten.
 * Calls that share a workspace must not overlap on the GPU.
 */
int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *out, float *lse,
                   int B, int H, int H_kv, int L_q, int L_k, int D, float scale,
                   int causal, int window_left, int window_right, int dtype,
                   int n_splits, void *workspace, size_t workspace_bytes,
                   cudaStream_t stream);

/*
 * fa_fwd_fp8_ex -- fa_fwd_fp8 with fa_fwd_ex's optional attention mask and
 * softmax statistics (same layouts and meaning; the mask's values are added
 * to the full-scale scores scale * descale_q * descale_k * q_i . k_j, and
 * softmax_max / softmax_sum refer to those scores).  Errors as fa_fwd_fp8
 * and fa_fwd_ex.
 */
int fa_fwd_fp8_ex(const void *q, const void *k, const void *v, void *out, float *lse,
                  float *softmax_max, float *softmax_sum, const void *mask, int mask_type,
                  long long mask_stride_b, long long mask_stride_h, long long mask_stride_q,
                  int B, int H, int H_kv, int L_q, int L_k, int D, float scale,
                  float descale_q, float descale_k, float descale_v, int causal,
                  int window_left, int window_right, cudaStream_t stream);

/*
 * fa_fwd_fp8_splitkv -- fa_fwd_fp8 computed in key slices as
 * fa_fwd_splitkv does (decoding over an fp8 key/value cache).  The slices'
 * partial outputs are fp32 in units of the V codes; the merge applies
 * descale_v and writes bf16.  Arguments as fa_fwd_fp8, plus n_splits,
 * workspace and workspace_bytes as fa_fwd_splitkv (the workspace size is
 * fa_splitkv_workspace_bytes(B, H, L_q, D, n_splits), the same as for
 * 16-bit inputs).  D must be 32, 64 or 128 (FA_ERR_HEADDIM otherwise).
 */
int fa_fwd_fp8_splitkv(const void *q, const void *k, const void *v, void *out, float *lse,
                       int B, int H, int H_kv, int L_q, int L_k, int D, float scale,
                       float descale_q, float descale_k, float descale_v, int causal,
                       int window_left, int window_right, int n_splits, void *workspace,
                       size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_bwd_workspace_bytes -- bytes of device workspace fa_bwd needs (0 if
 * the sizes are invalid): an fp32 dQ accumulator [B, H, L_q, D] and two
 * fp32 row vectors [B, H, roundup(L_q, 128)].
 */
size_t fa_bwd_workspace_bytes(int B, int H, int L_q, int D);

/*
 * fa_bwd -- exact attention backward on `stream` (asynchronous): the
 * gradients of sum(dout .* out) for out = fa_fwd(q, k, v, ...), with the
 * attention matrix recomputed from q, k and the forward's lse instead of
 * stored ("FlashAttention算法原理与性能优化实战" §1.2.3, recomputation; the
 * Triton FA2 walkthrough keeps the logsumexp for the backward pass).  With
 * P = softmax(scale q k^T + mask):
 *     dv = P^T dout,  dS = P .* (dout v^T - delta),  delta_i = dout_i . out_i,
 *     dq = scale dS k,  dk = scale dS^T q,
 * and for GQA the query heads that share a key/value head add into it.
 *
 *   q, out, dout  device, [B, H,    L_q, D], element type `dtype`
 *   k, v          device, [B, H_kv, L_k, D], element type `dtype`
 *   lse           device, [B, H, L_q] fp32: the forward's lse (-inf rows
 *                 see no key and get dq = 0)
 *   dq            device, [B, H,    L_q, D] written (RNE of fp32)
 *   dk, dv        device, [B, H_kv, L_k, D] written
 *   scale, causal, window_left, window_right, dtype: as fa_fwd, and the
 *                 same values the forward used
 *   workspace     device, 256-byte aligned, caller-owned, at least
 *                 fa_bwd_workspace_bytes(B, H, L_q, D) bytes
 *                 (FA_ERR_WORKSPACE if smaller); contents on entry do not
 *                 matter.  Calls that share a workspace must not overlap.
 * L_q == 0 writes dk = dv = 0; L_k == 0 writes dq = 0.  Pointers to tensors
 * with no elements may be NULL.  q, k, v, out, dout, dq, dk, dv need
 * 16-byte alignment, lse 4 bytes (FA_ERR_ALIGN).  Errors as fa_fwd.
 */
int fa_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout,
           const float *lse, void *dq, void *dk, void *dv, int B, int H, int H_kv, int L_q,
           int L_k, int D, float scale, int causal, int window_left, int window_right,
           int dtype, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_bwd_ex -- fa_bwd for a forward that used an attention mask (fa_fwd_ex):
 * P is recomputed with the same mask (same arguments, same reading: a
 * nonzero bool hides the key, a float is added to the scaled score; element
 * (b, h, i, j) at mask[b*mask_stride_b + h*mask_stride_h + i*mask_stride_q
 * + j]).  The mask itself gets no gradient.  Other arguments and errors as
 * fa_bwd; FA_ERR_ARG for a bad mask_type or a negative stride.
 */
int fa_bwd_ex(const void *q, const void *k, const void *v, const void *out, const void *dout,
              const float *lse, void *dq, void *dk, void *dv, const void *mask, int mask_type,
              long long mask_stride_b, long long mask_stride_h, long long mask_stride_q, int B,
              int H, int H_kv, int L_q, int L_k, int D, float scale, int causal,
              int window_left, int window_right, int dtype, void *workspace,
              size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_splitkv_auto_splits -- the number of key slices the library would pick
 * for fa_fwd_splitkv / fa_fwd_fp8_splitkv on the current device (dtype:
 * FA_F16, FA_BF16, or 2 for E4M3 inputs).  For decoding shapes (at most two
 * query rows per K/V head: L_q * H / H_kv <= 2, head dims 16, 32, 64, 128)
 * the forward runs on the CUDA cores over a persistent grid of one CTA per
 * SM, and the slices make (B * H_kv * slices) work items whose last round is
 * nearly full; otherwise the tensor-core kernel's query tiles and slices
 * fill waves of one CTA per SM.  Returns 1 for empty or invalid sizes.
 * This is a planning helper: a split count, not a result of the method.
 */
int fa_splitkv_auto_splits(int B, int H, int H_kv, int L_q, int L_k, int D, int dtype);

/*
 * fa_fwd_splitkv_static -- fa_fwd_splitkv with no workspace argument: the
 * partials live in a fixed scratch array inside the library (static device
 * memory, FA_STATIC_SCRATCH_BYTES per device).  The pages have no
 * counterpart to this entry point; it exists for callers that cannot
 * allocate device memory at the time they run attention: a process whose
 * device memory is all owned by another allocator (so that a cudaMalloc
 * beside it could fail or fragment it), a serving loop that must not take
 * cudaMalloc's implicit device synchronisation and unbounded latency after
 * start-up, or a plug-in that has no handle on its host's allocator.  Every
 * call, and the library itself, allocates nothing.
 *
 * Arguments as fa_fwd_splitkv without `workspace` / `workspace_bytes`.
 * Returns FA_ERR_SCRATCH, before touching the GPU, when
 * fa_splitkv_workspace_bytes(B, H, L_q, D, n_splits) exceeds
 * FA_STATIC_SCRATCH_BYTES (16 MiB: e.g. 32768 query rows x n_splits at
 * D = 128; lower n_splits to fit); other errors as fa_fwd_splitkv.
 *
 * Set-up: the first call on each device (with that device current) looks
 * up the scratch's device address once and caches it, keyed on the device's
 * context (a context made anew, e.g. after cudaDeviceReset, is looked up
 * again on its first call); make that first call before any stream
 * capture.  Nothing in the scratch has to start at zero:
 * every partial the merge reads is written earlier in the same call.
 * There is ONE scratch per device: calls whose work overlaps on the GPU
 * (different streams, or different host threads) race on it and corrupt
 * each other's results; serialise them (one stream, or events).
 */
#define FA_STATIC_SCRATCH_BYTES ((size_t)16 << 20)
int fa_fwd_splitkv_static(const void *q, const void *k, const void *v, void *out,
                          float *lse, int B, int H, int H_kv, int L_q, int L_k, int D,
                          float scale, int causal, int window_left, int window_right,
                          int dtype, int n_splits, cudaStream_t stream);

/*
 * fa_get_device_status -- synchronise `stream`, then read and clear the
 * device status word that the kernels set when a bounded wait gives up.
 * Returns FA_OK, FA_ERR_TIMEOUT, or FA_ERR_CUDA if the synchronisation or
 * the read failed.
 */
int fa_get_device_status(cudaStream_t stream);

/*
 * fa_selftest_wait_timeout -- exercise the device-side watchdog that every
 * kernel of this library relies on.  The pages have no counterpart; this
 * entry point exists so that the failure path can be tested on a GPU
 * without faulting it.  It enqueues one CTA of two warps on `stream`:
 *   warp 0 waits on an mbarrier phase that completes (one arrival), then on
 *          one that nothing completes; that wait gives up after the
 *          library's wait limit (1 s), raises the CTA's abort flag and sets
 *          the device status word, and the warp returns;
 *   warp 1 sleeps 0.5 s, then waits on the same never-completed phase and
 *          must give up as soon as warp 0 raises the abort flag, before its
 *          own limit.
 * `result` (device memory, 6 ints, written by the kernel):
 *   [0] 1 if the completed wait returned success, [1] 1 if the abandoned
 *   wait returned success (expected 0), [2] the abort flag afterwards
 *   (expected 1), [3] warp 0's abandoned wait in ms (about 1000), [4] 1 if
 *   warp 1's wait returned success (expected 0), [5] warp 1's wait in ms
 *   (about 500).
 * The kernel occupies one SM for about 1 s.  Afterwards
 * fa_get_device_status(stream) returns FA_ERR_TIMEOUT once (and clears
 * it); the context stays usable.  Returns FA_ERR_NULL for a NULL result,
 * FA_ERR_CUDA if the launch fails, else FA_OK.
 */
int fa_selftest_wait_timeout(int *result, cudaStream_t stream);

/* fa_status_string -- a static, human-readable name for a status code. */
const char *fa_status_string(int status);

/*
 * fa_version -- library version as major*10000 + minor*100 + patch.
 */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H */
