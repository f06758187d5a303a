/*
 * vla_attn.h -- C ABI of the B200 (sm_100a) self-attention core of a ViT /
 * SigLIP vision encoder.
 *
 * Operation.  For every image b, head h and query token i of a packed QKV
 * buffer, the library computes
 *
 *     o[b,i,h,:] = sum_j softmax_j( scale * q[b,i,h,:] . k[b,j,h,:] ) v[b,j,h,:]
 *
 * over all N tokens of the image (bidirectional, no mask, no dropout).  This
 * is the multi-head self-attention of the ViT backbone that the Pi0 Flash
 * Attention tutorial accelerates ("Pi0 VLA deployment tutorial: Flash
 * Attention for the vision encoder", section 1 for the operation and the
 * claim that the fused kernel keeps the output unchanged, section 3.2 for the
 * qkv linear feeding nn.MultiheadAttention / FlashMHA at inference, dropout 0).
 * The same layers are the ViT-L/14 tower of the "Pi0 VLA latency report on a
 * 16 GB GPU" (section 3.1) and the SigLIP tower of the Realtime-VLA write-up
 * (section 1.1.2).
 *
 * Data layout.
 *   q, k, v   point into ONE packed bf16 buffer laid out [B, N, 3, H, d]
 *             (what the encoder's qkv linear emits, viewed per head):
 *             k == q + H*d elements, v == q + 2*H*d elements, token stride
 *             3*H*d elements.  Any other relation is rejected.
 *   o         separate bf16 buffer [B, N, H, d] (= [B, N, H*d], the input of
 *             the output projection).
 *   Arithmetic: bf16 inputs, fp32 accumulation of Q K^T and P V on the tensor
 *   cores, fp32 online softmax, P rounded to bf16 before P V, O rounded to
 *   bf16 (nearest even) on store.
 *
 * Ownership.  The caller owns every buffer.  vla_attn_fwd allocates no memory,
 * never synchronises the host, and enqueues exactly one kernel on `stream`
 * (a cudaStream_t; NULL = the legacy default stream).  All pointers are device
 * pointers of the current device.
 *
 * Errors.  Argument errors are returned synchronously before anything is
 * enqueued.  A launch failure returns VLA_ATTN_ERR_CUDA.  Every wait inside
 * the kernel is bounded; a wait that runs out records a code in a device-side
 * status word, which vla_attn_last_device_status() reports.
 */
#ifndef VLA_ATTN_H_
#define VLA_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VLA_ATTN_OK = 0,
  VLA_ATTN_ERR_NULL = -1,        /* a required pointer is NULL */
  VLA_ATTN_ERR_SHAPE = -2,       /* B, N or H < 1, or q/k/v not the packed [B,N,3,H,d] relation */
  VLA_ATTN_ERR_UNSUPPORTED = -3, /* d not 64 or 72, or N above vla_attn_max_tokens(d) */
  VLA_ATTN_ERR_ALIGN = -4,       /* q or o not 16-byte aligned */
  VLA_ATTN_ERR_SCALE = -5,       /* scale not finite or not > 0 */
  VLA_ATTN_ERR_CUDA = -6,        /* a CUDA runtime / driver call failed */
  VLA_ATTN_ERR_TIMEOUT = -7,     /* a bounded in-kernel wait ran out (device status) */
  VLA_ATTN_ERR_DEVICE = -8,      /* current device is not sm_100 (B200 class) */
  VLA_ATTN_ERR_MEMORY = -9       /* a pointer is not device memory of the current device,
                                    or its allocation is too small for the shape */
} vla_attn_status;

/*
 * Attention forward on the packed QKV buffer (see the header comment).
 *   q, k, v  device pointers into one [B, N, 3, H, d] bf16 buffer (k = q + H*d,
 *            v = q + 2*H*d elements); q must be 16-byte aligned.
 *   o        device pointer to [B, N, H, d] bf16 output, 16-byte aligned; must
 *            not overlap the input.
 *   B        images (camera views x batch), >= 1.
 *   N        tokens per image (patches + CLS), 1 <= N <= vla_attn_max_tokens(d)
 *            (16384).  Up to 768 tokens for d=64 (560 for d=72) a head's K and
 *            V can stay in shared memory for all its query tiles; longer
 *            sequences, and batches of at least one head per SM whose heads
 *            have an odd number of 128-row query tiles (their tiles are then
 *            paired across heads), stream K/V blocks through the
 *            shared-memory ring per pair of query tiles (same result, more
 *            L2 traffic).
 *   H        heads, >= 1.
 *   d        head dimension, 64 (ViT-B/16, ViT-L/14) or 72 (SigLIP-So400m/14).
 *   scale    logit scale, usually 1/sqrt(d); finite and > 0.
 *   stream   cudaStream_t to enqueue on.
 * Returns VLA_ATTN_OK or a negative vla_attn_status.
 */
int vla_attn_fwd(const void* q, const void* k, const void* v, void* o,
                 int B, int N, int H, int d, float scale, void* stream);

/*
 * End-to-end variant for callers whose data live in host memory: copies the
 * packed [B, N, 3, H, d] bf16 input from `qkv_host` into the caller's device
 * buffer `qkv_dev`, runs vla_attn_fwd on it into `o_dev`, and copies the
 * [B, N, H, d] bf16 result back to `o_host`.  A batch of at least two chunks
 * (a chunk = the fewest whole images with one head per SM) is pipelined per
 * chunk: the input copies back to back on an internal copy-in stream of the
 * device (after the earlier work of `stream`), each chunk's kernel on
 * `stream` once its input has landed, its result copy on an internal
 * copy-out stream, so that copies in both directions and the kernels
 * overlap; `stream` then waits for both internal streams.  Smaller batches
 * use one copy per direction on `stream`.  Either way the results are those of
 * vla_attn_fwd on the whole batch, and the host result is valid once
 * `stream` has been synchronised.  Host buffers should be pinned
 * (cudaHostAlloc / cudaHostRegister) for the copies to be asynchronous.
 * Same argument rules and status codes as vla_attn_fwd; the device buffers are
 * range-checked (qkv_dev must hold 3*B*N*H*d and o_dev B*N*H*d bf16 elements
 * inside one device allocation each, and they must not overlap) before the
 * first copy is enqueued, so an argument error leaves nothing enqueued.
 * Allocates no memory;
 * the first pipelined call on a device creates the two internal streams and
 * five events, which live as long as the process.  Calls are serialised on a
 * library lock while they enqueue.
 */
int vla_attn_fwd_host(const void* qkv_host, void* o_host, void* qkv_dev, void* o_dev,
                      int B, int N, int H, int d, float scale, void* stream);

/*
 * Utility calls.  The pages describe the operation only; the status calls
 * below, the launch counter and the testing hooks are this library's own
 * plumbing and follow no passage of them.
 */

/* Human-readable text for a status code (static storage, never NULL). */
const char* vla_attn_strerror(int status);

/*
 * Synchronises `stream` and returns the device-side status of the kernels run
 * since the last reset: VLA_ATTN_OK, or VLA_ATTN_ERR_TIMEOUT if a bounded wait
 * ran out (the output of that launch is then undefined).  `site`, if non-NULL,
 * receives the code of the first wait that ran out (0 if none): 1-3 the TMA
 * producer (Q slot, K block, V block), 11-16 the tensor-core issuers (Q, K,
 * V, P, S read out, previous round's P V issued), 21-22 the softmax warps
 * (S, P V progress), 31 a drain wait, 41 the testing stall.  This extends the plain status call
 * vla_attn_last_device_status(stream) by the optional `site` out-parameter
 * (pass NULL for the plain form).  The status word is always kept; reading
 * it costs a stream synchronisation, so call it outside timed regions.
 */
int vla_attn_last_device_status(void* stream, int* site);

/* Clears the device-side status word of the current device (enqueued on `stream`). */
int vla_attn_reset_device_status(void* stream);

/* Largest N the kernels accept for head dimension d (0 if d is unsupported). */
int vla_attn_max_tokens(int d);

/* Number of kernels this library has launched in this process. */
uint64_t vla_attn_launch_count(void);

/*
 * Testing hook: bound (in nanoseconds) of every in-kernel wait for launches
 * that follow on this host thread's process; 0 restores the default (1 s).
 * A tiny bound makes waits run out on purpose so that the error path can be
 * exercised: the kernel then records VLA_ATTN_ERR_TIMEOUT, drains its own
 * copies and tensor-core work, frees its tensor memory and returns.
 */
void vla_attn_set_wait_limit_ns(uint64_t ns);

/*
 * Testing hook: while `enable` is non-zero, launches that follow make every
 * softmax warp wait on an mbarrier that nothing completes.  The wait runs out
 * after the bound set with vla_attn_set_wait_limit_ns (default 1 s), the
 * kernel records VLA_ATTN_ERR_TIMEOUT with site 41 and takes the error path
 * described there; the output of such a launch is undefined.  No fault or
 * trap is involved.  The attention pages describe no such hook.
 */
void vla_attn_set_test_stall(int enable);

/*
 * LayerNorm over the last dimension of M rows of width W (the norm before a
 * ViT block's qkv linear; "FluxVLA docs, inference acceleration", Triton fused
 * kernels: norm fusion):
 *   y[m,i] = (x[m,i] - mean_m) / sqrt(var_m + eps) * gamma[i] + beta[i],
 *   var_m the biased variance, statistics in fp32.
 *   x, y     device pointers, [M, W] bf16 row-major, 16-byte aligned; y may be
 *            x (in place) but must not otherwise overlap an input.
 *   gamma, beta  device pointers, [W] bf16, 16-byte aligned.
 *   W        a multiple of 8, at most 2048 (ViT-B 768, ViT-L 1024, SigLIP 1152).
 *   eps      finite, >= 0 (timm ViT and SigLIP use 1e-6).
 * Returns VLA_ATTN_OK or a negative status (same codes as vla_attn_fwd;
 * VLA_ATTN_ERR_SCALE for a bad eps).
 */
int vla_layernorm_fwd(const void* x, const void* gamma, const void* beta, void* y, int M, int W,
                      float eps, void* stream);

/*
 * Linear layer with bias and optional residual, weights in nn.Linear layout
 * (same page, section 3, CUDA custom operators: GEMM + bias (+ residual) in
 * one launch; the "Pi0 VLA deployment tutorial", section 3.2: the block's qkv
 * linear feeds the attention):
 *   y[m,n] = sum_k x[m,k] * w[n,k] + bias[n] + res[m,n]
 * One launch of the library's tcgen05 GEMM: bf16 in, fp32 accumulation in
 * tensor memory, bias and residual added in the fp32 epilogue, one rounding to
 * bf16 (nearest even).  For the qkv linear (N = 3 H d), y is the packed
 * [B, tokens, 3, H, d] input of vla_attn_fwd.
 *   x        device, [M, K] bf16 row-major.
 *   w        device, [N, K] bf16 row-major.
 *   bias     device [N] bf16, or NULL (no bias).
 *   res      device [M, N] bf16, or NULL (no residual); may equal y.
 *   y        device, [M, N] bf16 row-major; must not overlap x, w, bias, the
 *            workspace, or res unless it is res.
 *   K, N     multiples of 8.  All pointers 16-byte aligned.
 *   workspace, workspace_bytes  caller-owned device scratch (NULL with 0
 *            allowed).  When the output has too few 128-row tiles to fill the
 *            SMs and K is long enough for the split to pay (in practice K of
 *            several thousand and more with a few tiles; none of the encoder
 *            shapes), the K range is split and the parts' fp32 partial sums
 *            and per-tile arrival counters go here (the counters are cleared
 *            by a memset enqueued before the kernel); a shape is split only if
 *            its partial sums fit, otherwise it runs unsplit (same result up
 *            to fp32 summation order).  vla_linear_workspace_bytes() is enough
 *            for every split the library chooses.  The library allocates
 *            nothing.  Calls that share a workspace must be ordered on one
 *            stream.
 * Returns VLA_ATTN_OK or a negative status.
 */
int vla_linear_fwd(const void* x, const void* w, const void* bias, const void* res, void* y,
                   int M, int K, int N, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Residual add fused with LayerNorm ("FluxVLA docs, inference acceleration",
 * Triton fused kernels, norm fusion: residual add + LayerNorm in one kernel):
 *   s[m,i] = bf16(x[m,i] + r[m,i])      (sum in fp32, rounded to nearest even)
 *   y[m,i] = LayerNorm(s)[m,i]          (as vla_layernorm_fwd, on the stored s)
 * s is the new residual stream; normalising the stored bf16 values makes the
 * result identical to a separate add followed by vla_layernorm_fwd.
 *   x, r, s, y: [M, W] row-major bf16 device buffers; gamma, beta: [W] bf16.
 *   Each output may be exactly x or r (in-place stream update) or disjoint
 *   from them; s and y are disjoint; gamma and beta do not overlap an output.
 *   Shapes, alignment, eps and errors as vla_layernorm_fwd.  One launch on
 *   `stream`, no allocation, graph-capturable.
 */
int vla_add_layernorm_fwd(const void* x, const void* r, const void* gamma, const void* beta,
                          void* s, void* y, int M, int W, float eps, void* stream);

/*
 * Linear layer with bias and GELU in one launch, the first layer of the ViT
 * MLP (same page, Triton fused kernels: matrix multiply + bias + activation;
 * the activation is GELU in its tanh form,
 * a/2 (1 + tanh(sqrt(2/pi) (a + 0.044715 a^3))), as in SigLIP, evaluated with
 * the hardware tanh approximation in the GEMM's fp32 epilogue):
 *   y[m,n] = gelu(sum_k x[m,k] * w[n,k] + bias[n])
 *   Layout, alignment, workspace, bias (may be NULL), errors and the
 *   fp32-accumulate, bf16-output arithmetic as vla_linear_fwd; there is no
 *   residual input.  y must not overlap x, w, bias or the workspace.
 */
int vla_linear_gelu_fwd(const void* x, const void* w, const void* bias, void* y, int M, int K,
                        int N, void* workspace, size_t workspace_bytes, void* stream);

/* Recommended workspace size for vla_linear_fwd (bytes). */
size_t vla_linear_workspace_bytes(void);

/*
 * vla_linear_fwd without a caller workspace and without any allocation, for
 * callers that cannot allocate device memory (for instance code that runs
 * inside a stream capture, or a runtime that owns all device memory itself):
 * the split-K scratch is a file-scope device array of
 * vla_linear_static_workspace_bytes() (8 MiB) per device, whose address is
 * looked up with cudaGetSymbolAddress for each device and context the first
 * time it is used there.  A shape whose partial sums do not fit it runs
 * unsplit.  Arguments and results otherwise as vla_linear_fwd.
 *   Calls that overlap on the GPU (on different streams, or from different
 *   host threads without ordering) share the array and race; order them on
 *   one stream.  The array keeps the last call's contents; the arrival
 *   counters it holds are cleared by each call before its kernel.  The first
 *   call for a device (and context) does the set-up (the symbol lookup): make
 *   it before any stream capture that records later calls.
 * The pages have no counterpart of this entry point (a deployment variant of
 * the linear layer, not a step of the method).
 */
int vla_linear_fwd_static(const void* x, const void* w, const void* bias, const void* res, void* y,
                          int M, int K, int N, void* stream);

/* Size of the fixed workspace of vla_linear_fwd_static (bytes). */
size_t vla_linear_static_workspace_bytes(void);

#ifdef __cplusplus
}
#endif

#endif /* VLA_ATTN_H_ */
