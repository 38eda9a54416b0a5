// sla_internal.h -- shared declarations of the CUDA translation units of
// libsla.so: problem geometry, workspace layout and kernel launchers.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/sla.h"

namespace sla {

constexpr int kD = 128;                  // head dimension supported
constexpr int kBlkK = 64;                // key block
constexpr int kStateCols = kD * kD + kD; // h (d x d, stored [dim][channel]) then z (d)
constexpr int kStateChunk = 32;          // key blocks per partial sum of the global state

struct Geometry {
    int B, H, N, d, blk_q, blk_k;
    int BH, n_qb, n_kb, n_aw, k_sel, quant;  // n_aw: 32-bit words of a state-reduction mask row
    bool subtract;  // H_I = H_total - sum(selected); otherwise sum(unselected)
    int n_chunks;   // partial sums of the global state per head
};

struct Layout {
    size_t status, qbar, kbar, kpart, scores, idx, amask, q8, k8, qscale, kscale, kmean, states, partials, htot, hq, v16;
    size_t total;
};

// argument checks shared by every entry point that takes (B, H, N, d, blk_q, blk_k, topk)
sla_status check_shape(int B, int H, int N, int d, int blk_q, int blk_k, float topk);
Geometry make_geometry(int B, int H, int N, int d, int blk_q, int blk_k, float topk, int quant);
Layout make_layout(const Geometry &g);
int topk_count(int n_kb, float topk);

// ---- launchers (all asynchronous on `s`; return cudaGetLastError()) ----
// block means (and, when part != nullptr, per-CTA partial sums for launch_kmean)
int pool_parts(int nb);
cudaError_t launch_pool(const void *x, int BH, int N, int blk, int nb, double *mean, double *part, cudaStream_t s);
cudaError_t launch_kmean(const double *part, int BH, int N, int n_parts, float *kmean, cudaStream_t s);
cudaError_t launch_scores(const double *qbar, const double *kbar, const Geometry &g, double *scores,
                          cudaStream_t s);
cudaError_t launch_topk(const double *scores, const Geometry &g, int32_t *idx, uint32_t *bitmap,
                        uint32_t *amask, cudaStream_t s);
// INT8 (fp8 = 0) or FP8 e4m3 (fp8 = 1) codes and scales; with `bmean` (no smoothing) also the
// fp64 block means
cudaError_t launch_quant(const void *x, int BH, int N, int blk, int nb, const float *mean, int8_t *out,
                         float *scale, double *bmean, int fp8, cudaStream_t s);

// linear branch and fused attention (tcgen05)
cudaError_t launch_states(const void *k, const void *v, const Geometry &g, int phi, uint16_t *states,
                          float *partials, uint16_t *v16, int *status, cudaStream_t s);
cudaError_t launch_htot(const float *partials, const Geometry &g, float *htot, cudaStream_t s);
cudaError_t launch_state_reduce(const uint32_t *amask, const uint16_t *states, const float *htot,
                                const Geometry &g, float *hq, int *status, cudaStream_t s);
// v: bf16 V with quant = 1, the fp16 copy of V with quant = 0
cudaError_t launch_attention(const void *q, const void *k, const void *v, const int8_t *q8, const int8_t *k8,
                             const float *qscale, const float *kscale, const int32_t *idx, const float *hq,
                             const Geometry &g, int phi, void *out, int *status, cudaStream_t s);

// backward of the unquantised forward (sla_backward.cu); the workspace begins with the forward's
// quant = 0 layout
size_t backward_workspace_bytes(const Geometry &g);
cudaError_t launch_backward(const void *q, const void *k, const void *v, const void *dout, float *dq, float *dk,
                            float *dv, const Geometry &g, int phi, void *ws, cudaStream_t s);
// the softmax branch of the backward on the tensor cores (sla_bwd_tc.cu, as the linear branch's
// kernels below): the query side writes
// dq and the row statistics (max m, 1/l, D); the key side adds to dk, dv
cudaError_t launch_bwd_query_sparse(const void *q, const void *k, const void *v, const void *dout,
                                    const int32_t *idx, const float *kmean, const Geometry &g, float *dq,
                                    float *st_m, float *st_l, float *st_D, int *status, cudaStream_t s);
cudaError_t launch_bwd_key_sparse(const void *q, const void *k, const void *v, const void *dout,
                                  const uint32_t *selT, int n_awT, const float *st_m, const float *st_l,
                                  const float *st_D, const Geometry &g, float *dk, float *dv, int *status,
                                  cudaStream_t s);
// the linear branch of the backward on the tensor cores: the query side adds to dq and writes dH, dZ
// (fp32 and bf16); the key side writes dk, dv
cudaError_t launch_bwd_query_linear(const void *q, const void *dout, const float *hq, const Geometry &g, int phi,
                                    float *dq, float *dh32, uint16_t *dh16, int *status, cudaStream_t s);
cudaError_t launch_bwd_key_linear(const void *k, const void *v, const float *G, const Geometry &g, int phi, float *dk,
                                  float *dv, int *status, cudaStream_t s);
// TMA descriptor encoding (driver entry point fetched once through the runtime)
// W8A8 linear layer (sla_w8a8.cu)
cudaError_t launch_rowquant(const void *x, int rows, int cols, int norm, const float *gamma, float eps, int8_t *q,
                            float *scale, cudaStream_t s);
cudaError_t launch_w8a8_gemm(const int8_t *qx, const float *sx, const int8_t *qw, const float *sw, const float *bias,
                             int M, int N, int K, void *out, int *status, cudaStream_t s);
// run-time override of the bounded waits' budget, one setter per translation unit with waiting
// kernels (cycles; 0 = default), on the current device
cudaError_t set_wait_budget_attention(long long cycles);
cudaError_t set_wait_budget_linear(long long cycles);
cudaError_t set_wait_budget_w8a8(long long cycles);
cudaError_t set_wait_budget_bwd(long long cycles);
bool encode_tmap(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *base, const uint64_t *dims,
                 const uint64_t *strides_bytes /* rank-1 entries */, const uint32_t *box);

}  // namespace sla
