// sla_backward.cu -- gradients of the unquantised SageSLA forward with respect
// to q, k and v, for SLA fine-tuning (the jiqiren.org.cn TurboDiffusion
// article, 方法论: full attention is replaced by SLA and the pretrained model is
// fine-tuned for the sparsity; the "TurboDiffusion" summary page, 主要能力: SLA
// white-box training).  The block selection is piecewise constant in (q, k) and is held
// fixed; every other step is the exact chain rule of the forward:
//
//   sparse branch (row i, selected tokens j, s = q.k / sqrt(d), p = softmax(s),
//   os = sum p v):  dv_j += p_ij do_i;  ds_ij = p_ij (do_i.v_j - do_i.os_i);
//   dq_i += ds_ij k_j / sqrt(d);  dk_j += ds_ij q_i / sqrt(d).
//   linear branch (row i of query block I, f = phi(q_i), a = f H_I,
//   b = f.Z_I, ol = a / b, zero when b = 0):  da = do / b;
//   db = -(do.ol) / b;  dq_i += (H_I da + Z_I db) phi'(q_i);
//   dH_I = sum_i f (outer) da;  dZ_I = sum_i f db;  for key block J,
//   G_J = sum of dH_I (g_J of dZ_I) over the query blocks that did not select
//   J:  dk_j += (G_J v_j + g_J) phi'(k_j);  dv_j += G_J^T phi(k_j).
//
// Launch sequence (all on one stream):
//   1. the forward's block means, scores, top-k, key-block states and
//      per-query-block states H_I, Z_I (the forward's own kernels, quantisation
//      off), and the head's mean key mu (for the dq of the softmax branch);
//   2. the softmax branch's query side on the tensor cores (bwdq_kernel,
//      sla_bwd_tc.cu): the row statistics (max, sum, D = do.os) and its dq;
//   3. the linear branch's query side (bwd_qlin_kernel, sla_bwd_tc.cu): its dq
//      (added), and dH_I, dZ_I (fp32 and a bf16 copy);
//   4. the column sum of dH_I over the query blocks (for the subtract form) and
//      the transposed selection bits (key block J -> query blocks I);
//   5. G = A^T dH on the tensor cores: the forward's state-reduction kernel on
//      the transposed mask (same subtract / complement rule);
//   6. the linear branch's key side (bwd_klin_kernel): dk, dv from G_J, written;
//   7. the softmax branch's key side on the tensor cores (bwdk_kernel): its dk,
//      dv over the query blocks that selected the key block, added.
//
// Every product runs as a tcgen05 MMA with bf16 operands and fp32
// accumulation: the softmax branch's per-tile products (P and dS rounded to
// bf16) and the linear branch's d x d products (phi(Q), dA, H_I, G_J, V and
// phi(K) rounded to bf16).  Results are fp32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/sla.h"
#include "sla_internal.h"

namespace sla {
namespace {

// selected query blocks of every key block, as bits (and, for the state reduction in complement
// mode, the unselected ones)
__global__ void sel_transpose_kernel(const int32_t *__restrict__ idx, int n_qb, int n_kb, int k_sel, int n_awT,
                                     uint32_t *__restrict__ selT)
{
    const int bh = blockIdx.y;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n_qb * k_sel; e += gridDim.x * blockDim.x) {
        const int I = e / k_sel, J = __ldg(idx + (size_t)bh * n_qb * k_sel + e);
        atomicOr(selT + ((size_t)bh * n_kb + J) * n_awT + (I >> 5), 1u << (I & 31));
    }
}

__global__ void complement_kernel(const uint32_t *__restrict__ selT, size_t n_words, int n_awT, int n_qb,
                                  uint32_t *__restrict__ out)
{
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n_words; e += (size_t)gridDim.x * blockDim.x) {
        const int w = (int)(e % n_awT);
        const int valid = min(32, max(0, n_qb - 32 * w));
        const uint32_t m = valid == 32 ? 0xFFFFFFFFu : (1u << valid) - 1u;
        out[e] = ~selT[e] & m;
    }
}

struct BwdLayout {
    Layout fwd;
    size_t st_m, st_l, st_D, dh32, dh16, dhtot, selT, amaskT, G, total;
    int n_awT;
};

BwdLayout make_bwd_layout(const Geometry &g)
{
    BwdLayout L{};
    L.fwd = make_layout(g);
    L.n_awT = 2 * ((g.n_qb + 63) / 64);
    size_t off = L.fwd.total;
    auto take = [&](size_t bytes) { size_t o = off; off = (off + bytes + 255) / 256 * 256; return o; };
    const size_t BH = (size_t)g.BH;
    L.st_m = take(BH * g.N * sizeof(float));
    L.st_l = take(BH * g.N * sizeof(float));
    L.st_D = take(BH * g.N * sizeof(float));
    L.dh32 = take(BH * g.n_qb * (size_t)kStateCols * sizeof(float));
    L.dh16 = take(BH * g.n_qb * (size_t)kStateCols * sizeof(uint16_t));
    L.dhtot = take(BH * (size_t)kStateCols * sizeof(float));
    L.selT = take(BH * g.n_kb * (size_t)L.n_awT * sizeof(uint32_t));
    L.amaskT = g.subtract ? L.selT : take(BH * g.n_kb * (size_t)L.n_awT * sizeof(uint32_t));
    L.G = take(BH * g.n_kb * (size_t)kStateCols * sizeof(float));
    L.total = off;
    return L;
}

inline void *at(void *ws, size_t off) { return static_cast<uint8_t *>(ws) + off; }

}  // namespace

size_t backward_workspace_bytes(const Geometry &g) { return make_bwd_layout(g).total; }

cudaError_t launch_backward(const void *q, const void *k, const void *v, const void *dout, float *dq, float *dk,
                            float *dv, const Geometry &g, int phi, void *ws, cudaStream_t s)
{
    const BwdLayout L = make_bwd_layout(g);
    const Layout &F = L.fwd;
    int *status = static_cast<int *>(at(ws, F.status));
    double *qbar = static_cast<double *>(at(ws, F.qbar));
    double *kbar = static_cast<double *>(at(ws, F.kbar));
    double *kpart = static_cast<double *>(at(ws, F.kpart));
    float *kmean = static_cast<float *>(at(ws, F.kmean));
    double *scores = static_cast<double *>(at(ws, F.scores));
    int32_t *idx = static_cast<int32_t *>(at(ws, F.idx));
    uint32_t *amask = static_cast<uint32_t *>(at(ws, F.amask));
    uint16_t *states = static_cast<uint16_t *>(at(ws, F.states));
    float *partials = static_cast<float *>(at(ws, F.partials));
    float *htot = static_cast<float *>(at(ws, F.htot));
    float *hq = static_cast<float *>(at(ws, F.hq));
    float *st_m = static_cast<float *>(at(ws, L.st_m));
    float *st_l = static_cast<float *>(at(ws, L.st_l));
    float *st_D = static_cast<float *>(at(ws, L.st_D));
    float *dh32 = static_cast<float *>(at(ws, L.dh32));
    uint16_t *dh16 = static_cast<uint16_t *>(at(ws, L.dh16));
    float *dhtot = static_cast<float *>(at(ws, L.dhtot));
    uint32_t *selT = static_cast<uint32_t *>(at(ws, L.selT));
    uint32_t *amaskT = static_cast<uint32_t *>(at(ws, L.amaskT));
    float *G = static_cast<float *>(at(ws, L.G));
    cudaError_t e;
#define BWD_TRY(x) do { if ((e = (x)) != cudaSuccess) return e; } while (0)
    BWD_TRY(cudaMemsetAsync(status, 0, sizeof(int), s));
    // 1. the forward's selection and states (quantisation off), and the head's mean key
    BWD_TRY(launch_pool(q, g.BH, g.N, g.blk_q, g.n_qb, qbar, nullptr, s));
    BWD_TRY(launch_pool(k, g.BH, g.N, g.blk_k, g.n_kb, kbar, kpart, s));
    BWD_TRY(launch_kmean(kpart, g.BH, g.N, pool_parts(g.n_kb), kmean, s));
    BWD_TRY(launch_states(k, v, g, phi, states, partials, nullptr, status, s));
    BWD_TRY(launch_htot(partials, g, htot, s));
    BWD_TRY(launch_scores(qbar, kbar, g, scores, s));
    BWD_TRY(launch_topk(scores, g, idx, nullptr, amask, s));
    BWD_TRY(launch_state_reduce(amask, states, htot, g, hq, status, s));
    // 2. softmax branch, query side: row statistics and dq
    const int ks = g.k_sel;
    BWD_TRY(launch_bwd_query_sparse(q, k, v, dout, idx, kmean, g, dq, st_m, st_l, st_D, status, s));
    // 3. linear branch, query side: dq (added), dH_I, dZ_I
    BWD_TRY(launch_bwd_query_linear(q, dout, hq, g, phi, dq, dh32, dh16, status, s));
    // 4. column sum of dH over the query blocks; transposed selection bits
    {
        Geometry gh = g;
        gh.n_chunks = g.n_qb;
        BWD_TRY(launch_htot(dh32, gh, dhtot, s));
        BWD_TRY(cudaMemsetAsync(selT, 0, (size_t)g.BH * g.n_kb * L.n_awT * sizeof(uint32_t), s));
        if (ks > 0) {
            sel_transpose_kernel<<<dim3((g.n_qb * ks + 255) / 256, g.BH), 256, 0, s>>>(idx, g.n_qb, g.n_kb, ks,
                                                                                       L.n_awT, selT);
            BWD_TRY(cudaGetLastError());
        }
        if (!g.subtract) {
            const size_t n = (size_t)g.BH * g.n_kb * L.n_awT;
            complement_kernel<<<(unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096), 256, 0, s>>>(
                selT, n, L.n_awT, g.n_qb, amaskT);
            BWD_TRY(cudaGetLastError());
        }
    }
    // 5. G = A^T dH (the state reduction on the transposed mask)
    {
        Geometry gt = g;
        gt.n_qb = g.n_kb;
        gt.n_kb = g.n_qb;
        gt.n_aw = L.n_awT;
        BWD_TRY(launch_state_reduce(amaskT, dh16, dhtot, gt, G, status, s));
    }
    // 6. linear branch, key side: dk, dv written
    BWD_TRY(launch_bwd_key_linear(k, v, G, g, phi, dk, dv, status, s));
    // 7. softmax branch, key side: dk, dv added
    BWD_TRY(launch_bwd_key_sparse(q, k, v, dout, selT, L.n_awT, st_m, st_l, st_D, g, dk, dv, status, s));
#undef BWD_TRY
    return cudaSuccess;
}

}  // namespace sla
