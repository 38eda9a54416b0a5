/*
 * sla.h -- C ABI of libsla.so: the SageSLA attention forward (and its backward)
 * on B200 (sm_100a).
 *
 * SageSLA is Sparse-Linear Attention (SLA) with a SageAttention-style sparse
 * part, the attention used by TurboDiffusion's video DiT
 * ("TurboDiffusion技术架构解析：稀疏线性注意力应用实战" §2.1: standard
 * attention softmax(QK^T/sqrt(d))V, linear attention phi(Q)(phi(K)^T V) with
 * phi = ReLU or elu+1, and SLA keeping the top-k% most important key-value
 * pairs; "TurboDiffusion" summary page, 使用方式与安装: SageSLA is the
 * SageAttention-based fast SLA forward; "清华开源TurboDiffusion加速框架",
 * SageAttention与稀疏计算: INT8 low-bit attention on the tensor cores, about
 * 10% of the attention connections kept).
 *
 * What one call computes, per (batch b, head h):
 *   1. block means qbar_I (query blocks of blk_q tokens) and kbar_J (key blocks
 *      of blk_k tokens) over the valid tokens of each block;
 *   2. score s_IJ = qbar_I . kbar_J in fp64, accumulated over channels in order
 *      with one fused multiply-add per channel; per query block I the k_sel key
 *      blocks first in the order (score descending, block index ascending) are
 *      selected, k_sel = sla_topk_count(n_kb, topk);
 *   3. (quant = 1 or 2) K smoothed by its per-channel mean over all N tokens;
 *      Q and the smoothed K quantised with one fp32 scale per block: INT8 with
 *      quant = 1 (scale = amax/127, code = clamp(rint_even(x/scale), +-127)),
 *      FP8 e4m3 with quant = 2 (scale = amax/448, code = the e4m3 value
 *      nearest to x/scale, ties to even, saturating at +-448; no page names
 *      FP8 -- the SageAttention section speaks of INT8/INT4 -- so quant = 2 is
 *      an added mode on the same per-block scaling); every step in IEEE fp32;
 *   4. sparse branch: per query row, exact softmax attention over the tokens of
 *      the selected key blocks; logits (qhat.khat)*s_q*s_k/sqrt(d) with
 *      quant = 1 or 2 (INT8 MMA with int32 sums, or FP8 MMA with fp32 sums),
 *      (q.k)/sqrt(d) in bf16 x bf16 -> fp32 with quant = 0; P.V with P
 *      rounded to bf16 (quant = 1, 2) or to fp16 against an fp16 copy of V
 *      (quant = 0; V entries beyond +-65504 saturate), fp32 accumulation;
 *   5. linear branch over the unselected key blocks:
 *      phi(q)^T H_I / (phi(q) . Z_I), H_I = sum_{J unselected} phi(K_J)^T V_J,
 *      Z_I = sum_{J unselected} (column sums of phi(K_J)); phi acts on the raw
 *      Q and K; a zero denominator gives a zero linear output;
 *   6. out = sparse + linear, rounded to bf16.
 *
 * Beside the forward and its steps, the library exports the backward of the
 * unquantised forward (sla_backward: dq, dk, dv, for SLA fine-tuning), the
 * W8A8 INT8 linear layer with FusedNorm (sla_w8a8_*) and the block
 * permutations around a Ulysses all-to-all (sla_ulysses_permute); each is
 * described where it is declared.
 *
 * Layout: q, k, v, out are contiguous bf16 [B, H, N, d] (token index t-major).
 * Only d = 128, blk_k = 64 and blk_q in {64, 128} are supported.
 *
 * Memory: every pointer is caller-owned device memory (q, k, v, out, outputs
 * and the workspace), 16-byte aligned, except the host buffers of
 * sla_forward_host.  The library allocates no memory and keeps no per-call
 * global state (sla_forward and sla_forward_host create a few streams and
 * events of their own and release them before they return); calls on different
 * workspaces may run concurrently on different streams.  Calls that share one
 * workspace must be ordered (same stream or explicit events).
 *
 * Errors: arguments are validated before anything is enqueued; a bad argument
 * returns SLA_ERR_INVALID_ARG (null/misaligned pointer, negative size, topk
 * outside [0,1], phi/quant out of range), SLA_ERR_UNSUPPORTED (valid but not
 * implemented: d != 128, blk_k != 64, blk_q not 64/128) or SLA_ERR_WORKSPACE
 * (ws_bytes below sla_workspace_bytes).  A failed launch returns
 * SLA_ERR_CUDA.  Kernels never trap: every wait is bounded, and a device-side
 * failure (a wait that ran out, SLA_ERR_TIMEOUT) is recorded in a status word
 * inside the workspace, which sla_check reads.  Each call that takes a
 * workspace first clears that word (stream-ordered), so sla_check reports the
 * most recent call on that workspace.
 *
 * Streams: `stream` is a cudaStream_t passed as void*; NULL is the legacy
 * default stream.  All work is enqueued asynchronously on it.
 */
#ifndef SLA_H
#define SLA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SLA_API __attribute__((visibility("default")))
#else
#define SLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SLA_OK = 0,
    SLA_ERR_INVALID_ARG = 1,
    SLA_ERR_UNSUPPORTED = 2,
    SLA_ERR_WORKSPACE = 3,
    SLA_ERR_CUDA = 4,
    SLA_ERR_TIMEOUT = 5
} sla_status;

typedef enum { SLA_PHI_ELU1 = 0, SLA_PHI_RELU = 1 } sla_phi;

/* Library version string (static storage). */
SLA_API const char *sla_version(void);

/* Human-readable name of a status code (static storage; never NULL). */
SLA_API const char *sla_status_string(int status);

/* Selected key blocks per query block: floor(topk * n_kb + 1e-4) with topk
 * promoted to double, clamped to [0, n_kb].  Returns -1 if n_kb < 0 or topk
 * is not in [0, 1]. */
SLA_API int sla_topk_count(int n_kb, float topk);

/* Bytes of device workspace that sla_forward needs for this problem
 * (sla_block_mask and sla_quantize_qk need no more than this).  Returns 0
 * for arguments sla_forward would reject. */
SLA_API size_t sla_workspace_bytes(int B, int H, int N, int d, int blk_q, int blk_k, float topk, int quant);

/* Steps 1-2 only (pooled block scores and top-k selection).
 *   idx_out    int32 [B, H, n_qb, k_sel], each row ascending (required unless
 *              k_sel == 0).
 *   bitmap_out uint32 [B, H, n_qb, ceil(n_kb/32)] (nullable); bit J%32 of word
 *              J/32 is set iff key block J is selected.
 * The selection is bit-exact with the fp64 definition above. */
SLA_API sla_status sla_block_mask(const void *q_bf16, const void *k_bf16, int B, int H, int N, int d,
                          int blk_q, int blk_k, float topk, int32_t *idx_out, uint32_t *bitmap_out,
                          void *ws, size_t ws_bytes, void *stream);

/* Step 3 only (smoothing and INT8 quantisation).
 *   q_i8, k_i8  int8 [B, H, N, d] codes (k_i8 holds the smoothed K's codes)
 *   q_scale     fp32 [B, H, n_qb],  k_scale fp32 [B, H, n_kb]
 *   k_mean      fp32 [B, H, d] (nullable): the smoothing mean. */
SLA_API sla_status sla_quantize_qk(const void *q_bf16, const void *k_bf16, int B, int H, int N, int d,
                           int blk_q, int blk_k, int8_t *q_i8, int8_t *k_i8, float *q_scale,
                           float *k_scale, float *k_mean, void *ws, size_t ws_bytes, void *stream);

/* Step 3 with FP8 e4m3 codes (the codes sla_forward uses with quant = 2).
 *   q_fp8, k_fp8  uint8 [B, H, N, d] e4m3 bit patterns (k_fp8: the smoothed K)
 *   q_scale, k_scale, k_mean as for sla_quantize_qk (scales are amax / 448).
 * Codes are bit-exact with the fp32 definition above (a code that rounds to
 * zero keeps the sign of x). */
SLA_API sla_status sla_quantize_qk_fp8(const void *q_bf16, const void *k_bf16, int B, int H, int N, int d,
                               int blk_q, int blk_k, uint8_t *q_fp8, uint8_t *k_fp8, float *q_scale,
                               float *k_scale, float *k_mean, void *ws, size_t ws_bytes, void *stream);

/* The whole forward, steps 1-6.  quant: 0 = none, 1 = INT8, 2 = FP8 e4m3.
 * out: bf16 [B, H, N, d].  Stream-ordered on `stream`: its work starts after the
 * work queued there before the call and ends before the work queued after it.
 * Inside, the K side (K's block means, the linear states, K's smoothing mean and
 * codes) runs on a second stream that the call creates and releases, beside the Q
 * side and the block selection; not while `stream` is being captured into a
 * graph, where every step runs on `stream`. */
SLA_API sla_status sla_forward(const void *q, const void *k, const void *v, void *out, int B, int H, int N,
                       int d, int blk_q, int blk_k, float topk, int phi, int quant, void *ws,
                       size_t ws_bytes, void *stream);

/* The forward of sla_forward for callers whose Q, K, V and output are in HOST
 * memory.  The pages have no counterpart: this is a deployment variant of
 * sla_forward that keeps the host-device copies off the critical path.
 *
 * q_host, k_host, v_host: bf16 [B, H, N, d] in host memory; out_host: bf16
 * [B, H, N, d] in host memory, written.  Page-locked buffers (cudaHostAlloc,
 * cudaHostRegister) let the copies overlap the compute; pageable buffers give
 * the same result with the copies serialised by the driver.
 *
 * The B*H (batch, head) problems are independent.  The call takes them in
 * chunks of chunk_heads consecutive problems (the last chunk may be smaller)
 * and, for each chunk, copies its Q, K, V in on one stream, runs the forward
 * on a second and copies its output back on a third, so that the copy-in of
 * chunk c+1 and the copy-out of chunk c-1 overlap the forward of chunk c.
 * The output equals, bit for bit, that of one sla_forward over the whole
 * problem.
 *
 * dev: device memory of at least sla_forward_host_bytes(...) bytes, 16-byte
 * aligned, owned by the caller: the workspace of one chunk's forward at offset
 * 0, then two staging slots of Q, K, V and output for one chunk each.  The
 * status word is the workspace's: sla_check(dev, stream) reports the call.
 * The first chunk clears it, and later chunks keep an error an earlier chunk
 * recorded (they then exit early; the output is undefined).
 *
 * Ordering: the call's device work starts after the work already queued on
 * `stream`, and work queued on `stream` after the call starts after the last
 * copy-out, so out_host is complete once `stream` has been synchronised
 * (sla_check does that).  The host buffers must stay valid until then.  The
 * call creates its own three streams and 1 + 3*ceil(B*H/chunk_heads) events
 * and releases them before it returns (CUDA frees them when their work is
 * done); it allocates no memory.
 *
 * Errors: the shape checks of sla_forward; SLA_ERR_INVALID_ARG for a null host
 * pointer, chunk_heads < 1 or a null or misaligned dev; SLA_ERR_WORKSPACE when
 * dev_bytes is below sla_forward_host_bytes; SLA_ERR_CUDA when a stream, an
 * event or a copy cannot be created or queued (the call then waits for
 * whatever it had queued before returning).  sla_forward_host_bytes returns 0
 * for arguments that sla_forward_host would reject before any work. */
SLA_API size_t sla_forward_host_bytes(int B, int H, int N, int d, int blk_q, int blk_k, float topk, int quant,
                                      int chunk_heads);
SLA_API sla_status sla_forward_host(const void *q_host, const void *k_host, const void *v_host, void *out_host,
                                    int B, int H, int N, int d, int blk_q, int blk_k, float topk, int phi,
                                    int quant, int chunk_heads, void *dev, size_t dev_bytes, void *stream);

/* sla_block_mask for callers that cannot allocate device memory (for example
 * code inside a framework that owns the whole device-memory budget and hands
 * out no scratch buffers, or a latency-critical path where cudaMalloc's
 * implicit synchronisation is not acceptable).  The pages have no counterpart:
 * this is a deployment variant of the block-mask entry point.
 *
 * Same arguments, results and checks as sla_block_mask, without the
 * workspace: the scratch (block sums, scores, mask rows) lives in one
 * file-scope device array of sla_block_mask_noalloc_limit() bytes (16 MiB),
 * which every GPU that loads the library holds until the process exits.
 * Problems whose scratch would exceed it return SLA_ERR_WORKSPACE before any
 * launch.  The scratch is the sum of these regions, each rounded up to a
 * multiple of 256 bytes: 1024*B*H*n_qb and 1024*B*H*n_kb (fp64 block means),
 * 8*B*H*n_qb*n_kb (fp64 scores), 8*B*H*n_qb*ceil(n_kb/64) (mask rows), and
 * 4*B*H*n_qb only when k_sel == 0.  It allocates nothing.
 *
 * The first call on a device resolves the array's device address for that
 * device (cudaGetSymbolAddress, device current); make that first call before
 * any stream capture.  The address is kept for the life of the process: it
 * does not survive cudaDeviceReset of that device, so do not call this entry
 * point on a device after resetting it.  All calls share the one array: calls whose work
 * overlaps on the GPU (different streams, or different host threads without
 * ordering) race on it and must be serialised by the caller.  Nothing in the
 * array needs to start at zero: every value a call reads it wrote first. */
SLA_API sla_status sla_block_mask_noalloc(const void *q_bf16, const void *k_bf16, int B, int H, int N, int d,
                                          int blk_q, int blk_k, float topk, int32_t *idx_out,
                                          uint32_t *bitmap_out, void *stream);

/* Size in bytes of the static scratch array sla_block_mask_noalloc uses. */
SLA_API size_t sla_block_mask_noalloc_limit(void);

/* sla_forward with per-stage device timing: enqueues the same launches with a
 * CUDA event between stages, waits for them, and writes 7 floats to the host
 * array stage_ms: milliseconds of {Q quantisation (with the pooled Q means;
 * pooling alone when quant = 0), pooled K means + linear states,
 * scores + top-k, K smoothing + quantisation, per-query-block state,
 * attention, whole call}.  Blocks the
 * calling host thread until the call has finished on `stream`. */
SLA_API sla_status sla_forward_profile(const void *q, const void *k, const void *v, void *out, int B, int H, int N,
                                       int d, int blk_q, int blk_k, float topk, int phi, int quant, void *ws,
                                       size_t ws_bytes, void *stream, float *stage_ms);

/* ---- Backward, for SLA fine-tuning (the jiqiren.org.cn TurboDiffusion article,
 * 方法论: full attention is replaced by SLA and the pretrained model fine-tuned
 * for the sparsity; "TurboDiffusion" summary page, 主要能力: SLA white-box
 * training).
 *
 * Gradients of the unquantised forward (sla_forward with quant = 0) with
 * respect to q, k and v for the output gradient dout:
 *   q, k, v, dout  bf16 [B, H, N, d] (dout: dL/d out)
 *   dq, dk, dv     fp32 [B, H, N, d], overwritten (every element written)
 * The block selection is a piecewise-constant function of (q, k) and is held
 * fixed (the forward's own selection, recomputed); every other step is the
 * exact chain rule: the softmax gradient over the selected tokens, and the
 * linear branch's through phi(q) H_I / (phi(q) . Z_I) (a zero denominator gives
 * no gradient) and through the key-block states into k and v.  Arithmetic: the
 * forward's selection and states recomputed as in sla_forward; the sparse
 * branch's per-tile products on the tensor cores with bf16 operands (P and dS
 * rounded to bf16) and fp32 accumulation; the linear branch's products in
 * fp32; the state gradients summed over query blocks on the tensor cores in
 * bf16 x bf16 -> fp32.  Same shapes, limits and alignment as
 * sla_forward; phi as there.  ws: sla_backward_workspace_bytes bytes, 16-byte
 * aligned (its status word is read by sla_check).  Asynchronous on `stream`. */
SLA_API size_t sla_backward_workspace_bytes(int B, int H, int N, int d, int blk_q, int blk_k, float topk);
SLA_API sla_status sla_backward(const void *q_bf16, const void *k_bf16, const void *v_bf16, const void *dout_bf16,
                                float *dq, float *dk, float *dv, int B, int H, int N, int d, int blk_q, int blk_k,
                                float topk, int phi, void *ws, size_t ws_bytes, void *stream);

/* ---- W8A8 INT8 linear layer with FusedNorm ("清华开源TurboDiffusion加速框架",
 * W8A8 INT8量化: the linear layers' weights and activations quantised to 8-bit
 * integers on the INT8 units; "TurboDiffusion：让可视化视频生成效率提升200倍的
 * 加速引擎" §1: W8A8 with a FusedNorm operator).  This is not part of the
 * attention forward. */

/* Per-row symmetric INT8 quantisation of a bf16 matrix x [rows, cols]
 * (row-major): one fp32 scale per row, scale = amax / 127, code =
 * clamp(rint_even(y / scale), +-127), IEEE fp32.  With norm = 1 the row is
 * first RMS-normalised (FusedNorm): ms = (fp64 sum of x^2) / cols rounded to
 * fp32, r = 1 / sqrt(ms + eps), y = fp32(x * r) * gamma[c] (gamma nullable =
 * all ones; ignored when norm = 0).  Use it per token for activations and per
 * output channel (row of W [N, K]) for weights.
 *   q      int8 [rows, cols];  scale  fp32 [rows]
 * Requires cols % 8 == 0 and cols <= 16384 (else SLA_ERR_UNSUPPORTED); x, q and
 * gamma 16-byte aligned.  Codes are bit-exact with the definition above (the fp64
 * sum of squares is exact, as for the smoothing mean). */
SLA_API sla_status sla_w8a8_quantize(const void *x_bf16, int rows, int cols, int norm, const float *gamma,
                             float eps, int8_t *q, float *scale, void *stream);

/* Bytes of workspace sla_w8a8_linear needs (its status word, read by sla_check). */
SLA_API size_t sla_w8a8_workspace_bytes(void);

/* out[m][n] = bf16( float(sum_k qx[m][k] * qw[n][k]) * sx[m] * sw[n] + bias[n] )
 * with qx int8 [M, K] (per-token codes), sx fp32 [M], qw int8 [N, K] (per
 * output channel), sw fp32 [N], bias fp32 [N] (nullable), out bf16 [M, N]:
 * an INT8 tensor-core GEMM with int32 accumulation.  Requires K % 16 == 0 and
 * N % 8 == 0 (else SLA_ERR_UNSUPPORTED); qx, qw, out and ws 16-byte aligned. */
SLA_API sla_status sla_w8a8_linear(const int8_t *qx, const float *sx, const int8_t *qw, const float *sw,
                           const float *bias, int M, int N, int K, void *out_bf16, void *ws, size_t ws_bytes,
                           void *stream);

/* ---- Ulysses context parallelism (the "TurboDiffusion" summary page,
 * 主要能力: the training code supports Ulysses CP).  Each of P ranks holds
 * n_local = N / P consecutive tokens of every head; an all-to-all regroups them
 * into every token of H / P heads, the attention runs per head, and a second
 * all-to-all restores the token sharding.  This call does the block
 * permutation around each all-to-all (the exchange itself is the caller's, e.g.
 * NCCL's all_to_all_single on the [P][B][H/P][n_local][d] buffer, slice r to /
 * from rank r):
 *   mode 0  [B][H][n_local][d]        -> buffer   (tokens -> heads, send side)
 *   mode 1  buffer                    -> [B][H/P][P*n_local][d]  (receive side)
 *   mode 2  [B][H/P][P*n_local][d]    -> buffer   (heads -> tokens, send side)
 *   mode 3  buffer                    -> [B][H][n_local][d]      (receive side)
 * elem_bytes: 1, 2, 4 or 8.  H % P == 0; n_local * d * elem_bytes % 16 == 0 (else
 * SLA_ERR_UNSUPPORTED); src, dst 16-byte aligned and distinct. */
SLA_API sla_status sla_ulysses_permute(const void *src, void *dst, int B, int H, int P, int n_local, int d,
                               int elem_bytes, int mode, void *stream);

/* Diagnostics: sets, on the current device, the clock-cycle budget after which
 * every bounded wait in the library's kernels gives up (cycles > 0), or
 * restores the default of 10^9 cycles, about 0.5 s (cycles = 0).  A wait that
 * runs out records SLA_ERR_TIMEOUT in the call's status word and the kernel
 * unwinds: it stops issuing work, lets the copies and tensor-core operations
 * it already issued retire (those drain waits always keep the default budget),
 * releases its tensor memory and returns.  A budget of a few cycles therefore
 * makes any call whose kernels wait at all fail cleanly, which is how the
 * failure path is tested.  Process-wide per device and not ordered with
 * launches on other host threads: set it while no other call is being
 * enqueued.  Returns SLA_ERR_INVALID_ARG for cycles < 0, SLA_ERR_CUDA if the
 * setting could not be copied to the device.  The pages have no counterpart. */
SLA_API sla_status sla_set_wait_budget(long long cycles);

/* Synchronises `stream` and returns the device-side status word of `ws`
 * (SLA_OK, or SLA_ERR_TIMEOUT when a bounded wait ran out), or SLA_ERR_CUDA
 * if the synchronisation itself failed. */
SLA_API sla_status sla_check(void *ws, void *stream);

/* Byte offsets of the workspace's internal regions for this problem, for
 * inspection by tests: fills up to `n` entries of `offsets` in the order
 * {status, qbar, kbar, scores, idx, amask, q8, k8, qscale, kscale, kmean,
 *  states, partials, htot, hq, v16, kpart} and returns how many regions exist
 *  (qbar/kbar: fp64 pooled block means; kpart: fp64 partial sums of K for its
 *  per-channel mean).  A region
 * that a configuration does not use has offset (size_t)-1. */
SLA_API int sla_workspace_layout(int B, int H, int N, int d, int blk_q, int blk_k, float topk, int quant,
                         size_t *offsets, int n);

#ifdef __cplusplus
}
#endif

#endif /* SLA_H */
