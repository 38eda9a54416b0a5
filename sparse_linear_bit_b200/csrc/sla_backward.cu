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
//      sla_bwd_sparse.cu): the row statistics (max, sum, D = do.os) and its dq;
//   3. bwd_qlin_kernel, one CTA per (head, query block): the linear branch's
//      dq (added), and dH_I, dZ_I (fp32 and a bf16 copy);
//   4. the column sum of dH_I over the query blocks (for the subtract form) and
//      the transposed selection bits (key block J -> query blocks I);
//   5. G = A^T dH on the tensor cores: the forward's state-reduction kernel on
//      the transposed mask (same subtract / complement rule);
//   6. bwd_klin_kernel, one CTA per (head, key block): the linear key side from
//      G_J, written to dk, dv;
//   7. the softmax branch's key side on the tensor cores (bwdk_kernel): its dk,
//      dv over the query blocks that selected the key block, added.
//
// The softmax branch's per-tile products run as tcgen05 MMAs with bf16
// operands (P and dS rounded to bf16) and fp32 accumulation; the linear
// branch's d x d products run in fp32 on the CUDA cores.  Results are fp32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/sla.h"
#include "sla_internal.h"

namespace sla {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kRS = 68;          // 32-bit words per shared row of 128 bf16 (16-byte rows, conflict-free fragments)
constexpr int kGW = 129;         // floats per shared row of a 128 x 128 state tile
constexpr float kRsd = 0.08838834764831845f;  // 1 / sqrt(128)

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// element (r, c) of a shared tile of rows of 128 bf16, kRS words per row
__device__ __forceinline__ float tile_bf(const uint32_t *t, int r, int c)
{
    const uint32_t w = t[r * kRS + (c >> 1)];
    return (c & 1) ? bf_hi(w) : bf_lo(w);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float phi_f(float x, int phi)
{
    if (phi == 1) return fmaxf(x, 0.0f);
    return x > 0.0f ? x + 1.0f : __expf(fminf(x, 0.0f));
}

__device__ __forceinline__ float dphi_f(float x, int phi)
{
    if (phi == 1) return x > 0.0f ? 1.0f : 0.0f;
    return x > 0.0f ? 1.0f : __expf(fminf(x, 0.0f));
}

// Rows [row0, row0 + nrows) of a [., 128] bf16 matrix into the shared tile t (`rows` rows, kRS words
// each; rows past nrows are zero), and, when tt is given, its transpose: tt row c holds column c of
// the tile, two rows per 32-bit word (rs_t words per row).  `rows` is even.
__device__ __forceinline__ void load_tile(uint32_t *t, uint32_t *tt, int rs_t, const uint16_t *src, int row0,
                                          int nrows, int rows)
{
    const uint32_t *s = reinterpret_cast<const uint32_t *>(src) + (size_t)row0 * 64;
    for (int e = threadIdx.x; e < (rows >> 1) * 64; e += kBwdThreads) {
        const int pr = e >> 6, cw = e & 63, r = 2 * pr;
        const uint32_t w0 = r < nrows ? __ldg(s + (size_t)r * 64 + cw) : 0u;
        const uint32_t w1 = r + 1 < nrows ? __ldg(s + (size_t)(r + 1) * 64 + cw) : 0u;
        t[r * kRS + cw] = w0;
        t[(r + 1) * kRS + cw] = w1;
        if (tt) {
            tt[(2 * cw) * rs_t + pr] = __byte_perm(w0, w1, 0x5410);      // column 2cw of rows r, r+1
            tt[(2 * cw + 1) * rs_t + pr] = __byte_perm(w0, w1, 0x7632);  // column 2cw+1
        }
    }
}

// acc[i][j] += sum_k A(ty + 16 i, k) * B(k, tx + 16 j) over k < K, with ty = tid / 16, tx = tid % 16
// (fp32 on the CUDA cores: the linear branch's d x d products)
template <int TM, int TN, class FA, class FB>
__device__ __forceinline__ void gemm_acc(float (&acc)[TM][TN], int K, FA A, FB B)
{
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll 2
    for (int kk = 0; kk < K; ++kk) {
        float a[TM], b[TN];
#pragma unroll
        for (int i = 0; i < TM; ++i) a[i] = A(ty + 16 * i, kk);
#pragma unroll
        for (int j = 0; j < TN; ++j) b[j] = B(kk, tx + 16 * j);
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
}

// sum over the 16 threads (tx) that share a row group (a half warp)
__device__ __forceinline__ float hw_sum(float x)
{
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

struct QlinSmem {
    uint32_t q[128 * kRS];    // Q rows of the query block
    uint32_t dO[128 * kRS];   // dO rows
    float ht[128 * kGW];      // H_I^T
    float z[128], binv[128], db[128];
};

// ---------------------------------------------------------------------------
// step 3: the linear branch's query side, one CTA per (head, query block): dq += (H_I da + Z_I db)
// phi'(q) (dq holds the softmax branch's part), and dH_I, dZ_I for the key side
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_qlin_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ dout, const float *__restrict__ hq,
                int N, int blk_q, int n_qb, int phi, float *__restrict__ dq, float *__restrict__ dh32,
                uint16_t *__restrict__ dh16)
{
    extern __shared__ uint8_t smem_raw[];
    QlinSmem &sm = *reinterpret_cast<QlinSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int I = blockIdx.x, bh = blockIdx.y;
    const int i0 = I * blk_q, rows = min(blk_q, N - i0);  // valid rows of this query block
    const size_t head = (size_t)bh * N * 128;
    load_tile(sm.q, nullptr, 0, q + head, i0, rows, 128);
    load_tile(sm.dO, nullptr, 0, dout + head, i0, rows, 128);

    // ---- linear branch: H_I^T (stored [dim e][channel c]) and Z_I of this query block
    auto Qa = [&](int r, int c) { return tile_bf(sm.q, r, c); };
    auto dOa = [&](int r, int c) { return tile_bf(sm.dO, r, c); };
    float *ht = sm.ht;
    const float *hrow = hq + ((size_t)bh * n_qb + I) * kStateCols;
    for (int w = tid; w < 128 * 128; w += kBwdThreads) ht[(w >> 7) * kGW + (w & 127)] = __ldg(hrow + w);
    if (tid < 128) sm.z[tid] = __ldg(hrow + 128 * 128 + tid);
    __syncthreads();
    if (tid < 128) {  // 1 / b_i with b_i = phi(q_i).Z_I (0: no linear output, no gradient)
        float b = 0.0f;
        for (int c = 0; c < 128; ++c) b = fmaf(phi_f(Qa(tid, c), phi), sm.z[c], b);
        sm.binv[tid] = (tid < rows && b != 0.0f) ? 1.0f / b : 0.0f;
    }
    __syncthreads();
    auto Fa = [&](int r, int c) { return phi_f(Qa(r, c), phi); };
    auto HTt = [&](int c, int e) { return ht[e * kGW + c]; };  // B(c, e) = H[c][e] = H^T[e][c]
    auto HTr = [&](int e, int c) { return ht[e * kGW + c]; };  // B(e, c) = H^T[e][c]
    auto DAa = [&](int r, int e) { return dOa(r, e) * sm.binv[r]; };
    {
        float A[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) A[i][j] = 0.0f;
        gemm_acc<8, 8>(A, 128, Fa, HTt);  // a = phi(q) H_I
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int rr = ty + 16 * i;
            float part = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) part += dOa(rr, tx + 16 * j) * A[i][j];
            const float dot = hw_sum(part), bi = sm.binv[rr];
            if (tx == 0) sm.db[rr] = -dot * bi * bi;  // -(do.ol) / b with ol = a / b
        }
    }
    __syncthreads();
    {
        float dF[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) dF[i][j] = 0.0f;
        gemm_acc<8, 8>(dF, 128, DAa, HTr);  // H_I da
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int rr = ty + 16 * i;
            if (rr >= rows) continue;
            float *dst = dq + head + (size_t)(i0 + rr) * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c = tx + 16 * j;
                dst[c] += (dF[i][j] + sm.z[c] * sm.db[rr]) * dphi_f(Qa(rr, c), phi);
            }
        }
    }
    {
        // dH_I^T[e][c] = sum_i da_i[e] phi(q_i)[c]; dZ_I[c] = sum_i db_i phi(q_i)[c]
        float dH[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) dH[i][j] = 0.0f;
        gemm_acc<8, 8>(dH, 128, [&](int e, int r) { return DAa(r, e); }, [&](int r, int c) { return Fa(r, c); });
        float *d32 = dh32 + ((size_t)bh * n_qb + I) * kStateCols;
        uint16_t *d16 = dh16 + ((size_t)bh * n_qb + I) * kStateCols;
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int e = ty + 16 * i, c = tx + 16 * j;
                d32[e * 128 + c] = dH[i][j];
                d16[e * 128 + c] = __bfloat16_as_ushort(__float2bfloat16_rn(dH[i][j]));
            }
        if (tid < 128) {
            float s = 0.0f;
            for (int r = 0; r < 128; ++r) s = fmaf(sm.db[r], Fa(r, tid), s);
            d32[128 * 128 + tid] = s;
            d16[128 * 128 + tid] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
        }
    }
}

struct KlinSmem {
    uint32_t k[64 * kRS];   // K rows of the key block
    uint32_t v[64 * kRS];   // V rows
    float gt[128 * kGW];    // G_J^T
    float g[128];
};

// ---------------------------------------------------------------------------
// step 6: the linear branch's key side, one CTA per (head, key block)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_klin_kernel(const uint16_t *__restrict__ k, const uint16_t *__restrict__ v, const float *__restrict__ G, int N,
                int n_kb, int phi, float *__restrict__ dk, float *__restrict__ dv)
{
    extern __shared__ uint8_t smem_raw[];
    KlinSmem &sm = *reinterpret_cast<KlinSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int J = blockIdx.x, bh = blockIdx.y;
    const int t0 = J * 64, kv = min(64, N - t0);
    const size_t head = (size_t)bh * N * 128;

    load_tile(sm.k, nullptr, 0, k + head, t0, kv, 64);
    load_tile(sm.v, nullptr, 0, v + head, t0, kv, 64);
    float *gt = sm.gt;
    const float *grow = G + ((size_t)bh * n_kb + J) * kStateCols;
    for (int w = tid; w < 128 * 128; w += kBwdThreads) gt[(w >> 7) * kGW + (w & 127)] = __ldg(grow + w);
    if (tid < 128) sm.g[tid] = __ldg(grow + 128 * 128 + tid);
    __syncthreads();

    auto Ka = [&](int j, int c) { return tile_bf(sm.k, j, c); };
    auto Va = [&](int j, int e) { return tile_bf(sm.v, j, e); };
    auto GTr = [&](int e, int c) { return gt[e * kGW + c]; };  // B(e, c) = G^T[e][c]
    auto GTt = [&](int c, int e) { return gt[e * kGW + c]; };  // B(c, e) = G[c][e]

    // ---- linear key side (fp32): dk = (G_J v_j + g_J) phi'(k_j); dv = G_J^T phi(k_j), written
    //      here and completed by the softmax branch's key side
    {
        float T[4][8], L[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) T[i][j] = L[i][j] = 0.0f;
        gemm_acc<4, 8>(T, 128, Va, GTr);
        gemm_acc<4, 8>(L, 128, [&](int j, int c) { return phi_f(Ka(j, c), phi); }, GTt);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int jj = ty + 16 * i;
            if (jj >= kv) continue;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c = tx + 16 * j;
                dk[head + (size_t)(t0 + jj) * 128 + c] = (T[i][j] + sm.g[c]) * dphi_f(Ka(jj, c), phi);
                dv[head + (size_t)(t0 + jj) * 128 + c] = L[i][j];
            }
        }
    }
}

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
    {
        const size_t smem = sizeof(QlinSmem) + 16;
        BWD_TRY(cudaFuncSetAttribute(bwd_qlin_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        bwd_qlin_kernel<<<dim3(g.n_qb, g.BH), kBwdThreads, smem, s>>>(
            static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(dout), hq, g.N, g.blk_q, g.n_qb, phi, dq,
            dh32, dh16);
        BWD_TRY(cudaGetLastError());
    }
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
    {
        const size_t smem = sizeof(KlinSmem) + 16;
        BWD_TRY(cudaFuncSetAttribute(bwd_klin_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        bwd_klin_kernel<<<dim3(g.n_kb, g.BH), kBwdThreads, smem, s>>>(
            static_cast<const uint16_t *>(k), static_cast<const uint16_t *>(v), G, g.N, g.n_kb, phi, dk, dv);
        BWD_TRY(cudaGetLastError());
    }
    // 7. softmax branch, key side: dk, dv added
    BWD_TRY(launch_bwd_key_sparse(q, k, v, dout, selT, L.n_awT, st_m, st_l, st_D, g, dk, dv, status, s));
#undef BWD_TRY
    return cudaSuccess;
}

}  // namespace sla
