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
//      off);
//   2. bwd_query_kernel, one CTA per (head, query block): online-softmax
//      recompute of p and os over the selected blocks, the row statistics
//      (max, sum, D = do.os) for step 5, dq of both branches, and dH_I, dZ_I
//      (fp32 and a bf16 copy);
//   3. the column sum of dH_I over the query blocks (for the subtract form) and
//      the transposed selection bits (key block J -> query blocks I);
//   4. G = A^T dH on the tensor cores: the forward's state-reduction kernel on
//      the transposed mask (same subtract / complement rule);
//   5. bwd_key_kernel, one CTA per (head, key block): the linear key side from
//      G_J, then dk, dv of the sparse branch over the query blocks that
//      selected J (no atomics: each CTA owns its key block's rows).
//
// The per-tile products of the sparse branch (Q.K^T, P.V, dO.V^T, dS.K,
// P^T dO, dS^T Q) run on the tensor cores as warp-level bf16 MMAs with fp32
// accumulation; P and dS enter them rounded to bf16.  The linear branch's
// d x d products run in fp32 on the CUDA cores.  Results are fp32.
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
constexpr int kRS64 = 36;        // 32-bit words per shared row of 64 bf16
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

// ---- warp-level bf16 tensor-core products (mma.sync m16n8k16, fp32 accumulation).  Fragments are
// read from "k-major" shared tiles (row = the M or N index, two consecutive K elements per word).
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragment: rows m0..m0+15, K columns k0..k0+15
__device__ __forceinline__ void frag_a(const uint32_t *t, int rs, int m0, int k0, uint32_t (&a)[4])
{
    const int lane = threadIdx.x & 31;
    const uint32_t *p = t + (m0 + (lane >> 2)) * rs + (k0 >> 1) + (lane & 3);
    a[0] = p[0];
    a[1] = p[8 * rs];
    a[2] = p[4];
    a[3] = p[8 * rs + 4];
}

// acc[nt] (n-tile nt: N columns n0 + 8 nt ..) += A(m0.., 0..K) * B(0..K, n0 + 8 nt ..), B stored [n][k]
template <int NT>
__device__ __forceinline__ void warp_gemm(float (&acc)[NT][4], const uint32_t *ta, int rsa, int m0,
                                          const uint32_t *tb, int rsb, int n0, int K)
{
    const int lane = threadIdx.x & 31;
    const uint32_t *pb = tb + (n0 + (lane >> 2)) * rsb + (lane & 3);
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t a[4];
        frag_a(ta, rsa, m0, k0, a);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint32_t *q = pb + 8 * nt * rsb + (k0 >> 1);
            mma16816(acc[nt], a, q[0], q[4]);
        }
    }
}

// acc[nt] += P * B for P held as the fp32 accumulators of an m16 x n64 product (8 n-tiles), used as the
// A operand over K = 64 (the accumulator layout of two n-tiles is the A layout of one k-step)
template <int NT>
__device__ __forceinline__ void warp_gemm_regs(float (&acc)[NT][4], const float (&p)[8][4], const uint32_t *tb,
                                               int rsb, int n0)
{
    const int lane = threadIdx.x & 31;
    const uint32_t *pb = tb + (n0 + (lane >> 2)) * rsb + (lane & 3);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const uint32_t a[4] = {pack_bf16(p[2 * kk][0], p[2 * kk][1]), pack_bf16(p[2 * kk][2], p[2 * kk][3]),
                               pack_bf16(p[2 * kk + 1][0], p[2 * kk + 1][1]),
                               pack_bf16(p[2 * kk + 1][2], p[2 * kk + 1][3])};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint32_t *q = pb + 8 * nt * rsb + 8 * kk;
            mma16816(acc[nt], a, q[0], q[4]);
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

// reductions over the 16 threads (tx) that share a row group (a half warp), and over a quad
__device__ __forceinline__ float hw_sum(float x)
{
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float quad_max(float x)
{
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
    return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}
__device__ __forceinline__ float quad_sum(float x)
{
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

struct QuerySmem {
    uint32_t q[128 * kRS];    // Q rows of the query block
    uint32_t dO[128 * kRS];   // dO rows
    // key-block tiles; the linear part reuses this region for H_I^T (128 x kGW floats)
    uint32_t k[64 * kRS];     // K rows (B of Q.K^T)
    uint32_t kt[128 * kRS64]; // K^T (B of dS.K)
    uint32_t v[64 * kRS];     // V rows (B of dO.V^T)
    uint32_t vt[128 * kRS64]; // V^T (B of P.V)
    float z[128], binv[128], db[128];
};
static_assert(sizeof(uint32_t) * (2 * 64 * kRS + 2 * 128 * kRS64) >= sizeof(float) * 128 * kGW,
              "H_I^T fits in the key-block region");

// ---------------------------------------------------------------------------
// step 2: one CTA per (head, query block); warp w owns query rows 16w..16w+15 of the
// sparse products (rows g and g+8 of each fragment: r0, r1)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_query_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, const uint16_t *__restrict__ v,
                 const uint16_t *__restrict__ dout, const int32_t *__restrict__ idx, const float *__restrict__ hq,
                 int N, int blk_q, int n_qb, int k_sel, int phi, float *__restrict__ dq, float *__restrict__ st_m,
                 float *__restrict__ st_l, float *__restrict__ st_D, float *__restrict__ dh32,
                 uint16_t *__restrict__ dh16)
{
    extern __shared__ uint8_t smem_raw[];
    QuerySmem &sm = *reinterpret_cast<QuerySmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int warp = tid >> 5, lane = tid & 31, tq = lane & 3;
    const int r0 = 16 * warp + (lane >> 2), r1 = r0 + 8;
    const int I = blockIdx.x, bh = blockIdx.y;
    const int i0 = I * blk_q, rows = min(blk_q, N - i0);  // valid rows of this query block
    const size_t head = (size_t)bh * N * 128;
    const int32_t *sel = idx + ((size_t)bh * n_qb + I) * k_sel;

    load_tile(sm.q, nullptr, 0, q + head, i0, rows, 128);
    load_tile(sm.dO, nullptr, 0, dout + head, i0, rows, 128);

    // ---- sparse branch, pass 1: online softmax, os = sum p v, row statistics
    float O[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.0f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;
    for (int r = 0; r < k_sel; ++r) {
        const int t0 = __ldg(sel + r) * 64, kv = min(64, N - t0);
        __syncthreads();
        load_tile(sm.k, nullptr, 0, k + head, t0, kv, 64);
        load_tile(sm.v, sm.vt, kRS64, v + head, t0, kv, 64);
        __syncthreads();
        float s[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.0f;
        warp_gemm<8>(s, sm.q, kRS, 16 * warp, sm.k, kRS, 0, 128);
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const bool ok = 8 * n + 2 * tq + h < kv;
                s[n][h] = ok ? s[n][h] * kRsd : -INFINITY;
                s[n][2 + h] = ok ? s[n][2 + h] * kRsd : -INFINITY;
                mx0 = fmaxf(mx0, s[n][h]);
                mx1 = fmaxf(mx1, s[n][2 + h]);
            }
        const float mn0 = fmaxf(m0, quad_max(mx0)), mn1 = fmaxf(m1, quad_max(mx1));
        const float al0 = __expf(m0 - mn0), al1 = __expf(m1 - mn1);  // 0 while m = -inf
        float sum0 = 0.0f, sum1 = 0.0f;
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                s[n][h] = __expf(s[n][h] - mn0);
                s[n][2 + h] = __expf(s[n][2 + h] - mn1);
                sum0 += s[n][h];
                sum1 += s[n][2 + h];
            }
        l0 = l0 * al0 + quad_sum(sum0);
        l1 = l1 * al1 + quad_sum(sum1);
        m0 = mn0;
        m1 = mn1;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            O[n][0] *= al0; O[n][1] *= al0;
            O[n][2] *= al1; O[n][3] *= al1;
        }
        warp_gemm_regs<16>(O, s, sm.vt, kRS64, 0);  // O += P V
    }
    const float il0 = l0 > 0.0f ? 1.0f / l0 : 0.0f, il1 = l1 > 0.0f ? 1.0f / l1 : 0.0f;
    float D0 = 0.0f, D1 = 0.0f;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const uint32_t w0 = sm.dO[r0 * kRS + 4 * n + tq], w1 = sm.dO[r1 * kRS + 4 * n + tq];
        D0 += bf_lo(w0) * O[n][0] + bf_hi(w0) * O[n][1];
        D1 += bf_lo(w1) * O[n][2] + bf_hi(w1) * O[n][3];
    }
    D0 = quad_sum(D0) * il0;
    D1 = quad_sum(D1) * il1;
    if (tq == 0) {
        if (r0 < rows) {
            st_m[(size_t)bh * N + i0 + r0] = m0;
            st_l[(size_t)bh * N + i0 + r0] = il0;
            st_D[(size_t)bh * N + i0 + r0] = D0;
        }
        if (r1 < rows) {
            st_m[(size_t)bh * N + i0 + r1] = m1;
            st_l[(size_t)bh * N + i0 + r1] = il1;
            st_D[(size_t)bh * N + i0 + r1] = D1;
        }
    }

    // ---- sparse branch, pass 2: dq = sum_j p (do.v_j - D) k_j / sqrt(d)
    float dQ[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) dQ[n][0] = dQ[n][1] = dQ[n][2] = dQ[n][3] = 0.0f;
    for (int r = 0; r < k_sel; ++r) {
        const int t0 = __ldg(sel + r) * 64, kv = min(64, N - t0);
        __syncthreads();
        load_tile(sm.k, sm.kt, kRS64, k + head, t0, kv, 64);
        load_tile(sm.v, nullptr, 0, v + head, t0, kv, 64);
        __syncthreads();
        float s[8][4], dp[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.0f;
        warp_gemm<8>(s, sm.q, kRS, 16 * warp, sm.k, kRS, 0, 128);
        warp_gemm<8>(dp, sm.dO, kRS, 16 * warp, sm.v, kRS, 0, 128);
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const bool ok = 8 * n + 2 * tq + h < kv;
                const float p0 = ok ? __expf(s[n][h] * kRsd - m0) * il0 : 0.0f;
                const float p1 = ok ? __expf(s[n][2 + h] * kRsd - m1) * il1 : 0.0f;
                s[n][h] = p0 * (dp[n][h] - D0) * kRsd;
                s[n][2 + h] = p1 * (dp[n][2 + h] - D1) * kRsd;
            }
        warp_gemm_regs<16>(dQ, s, sm.kt, kRS64, 0);  // dq += dS K
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const int c = 8 * n + 2 * tq;
        if (r0 < rows) *reinterpret_cast<float2 *>(dq + head + (size_t)(i0 + r0) * 128 + c) = make_float2(dQ[n][0], dQ[n][1]);
        if (r1 < rows) *reinterpret_cast<float2 *>(dq + head + (size_t)(i0 + r1) * 128 + c) = make_float2(dQ[n][2], dQ[n][3]);
    }
    __syncthreads();  // the sparse dq rows are written; the key-block region is free

    // ---- linear branch: H_I^T (stored [dim e][channel c]) and Z_I of this query block
    auto Qa = [&](int r, int c) { return tile_bf(sm.q, r, c); };
    auto dOa = [&](int r, int c) { return tile_bf(sm.dO, r, c); };
    float *ht = reinterpret_cast<float *>(sm.k);
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

struct KeySmem {
    uint32_t k[64 * kRS];      // K rows (B of Q.K^T)
    uint32_t v[64 * kRS];      // V rows (B of dO.V^T)
    uint32_t pt[64 * kRS];     // P^T: row j holds P[.][j] over the query rows (A of P^T dO)
    uint32_t dst[64 * kRS];    // dS^T (A of dS^T Q)
    // query-block tiles; the linear key side uses this region first for G_J^T (128 x kGW floats)
    uint32_t q[128 * kRS];     // Q rows (A of Q.K^T)
    uint32_t qt[128 * kRS];    // Q^T (B of dS^T Q)
    uint32_t dO[128 * kRS];    // dO rows (A of dO.V^T)
    uint32_t dOt[128 * kRS];   // dO^T (B of P^T dO)
    float g[128], m[128], l[128], D[128];
};
static_assert(sizeof(uint32_t) * 4 * 128 * kRS >= sizeof(float) * 128 * kGW, "G_J^T fits in the query region");

// ---------------------------------------------------------------------------
// step 5: one CTA per (head, key block).  Q.K^T and dO.V^T: warp w owns query rows 16w..;
// P^T dO and dS^T Q: warp w owns key rows 16 (w % 4).. and dims / channels 64 (w / 4)..
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_key_kernel(const uint16_t *__restrict__ q, const uint16_t *__restrict__ k, const uint16_t *__restrict__ v,
               const uint16_t *__restrict__ dout, const uint32_t *__restrict__ selT, int n_awT,
               const float *__restrict__ G, const float *__restrict__ st_m, const float *__restrict__ st_l,
               const float *__restrict__ st_D, int N, int blk_q, int n_qb, int n_kb, int phi,
               float *__restrict__ dk, float *__restrict__ dv)
{
    extern __shared__ uint8_t smem_raw[];
    KeySmem &sm = *reinterpret_cast<KeySmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int warp = tid >> 5, lane = tid & 31, tq = lane & 3;
    const int J = blockIdx.x, bh = blockIdx.y;
    const int t0 = J * 64, kv = min(64, N - t0);
    const size_t head = (size_t)bh * N * 128;

    load_tile(sm.k, nullptr, 0, k + head, t0, kv, 64);
    load_tile(sm.v, nullptr, 0, v + head, t0, kv, 64);
    float *gt = reinterpret_cast<float *>(sm.q);
    const float *grow = G + ((size_t)bh * n_kb + J) * kStateCols;
    for (int w = tid; w < 128 * 128; w += kBwdThreads) gt[(w >> 7) * kGW + (w & 127)] = __ldg(grow + w);
    if (tid < 128) sm.g[tid] = __ldg(grow + 128 * 128 + tid);
    __syncthreads();

    auto Ka = [&](int j, int c) { return tile_bf(sm.k, j, c); };
    auto Va = [&](int j, int e) { return tile_bf(sm.v, j, e); };
    auto GTr = [&](int e, int c) { return gt[e * kGW + c]; };  // B(e, c) = G^T[e][c]
    auto GTt = [&](int c, int e) { return gt[e * kGW + c]; };  // B(c, e) = G[c][e]

    // ---- linear key side (fp32): dk = (G_J v_j + g_J) phi'(k_j); dv = G_J^T phi(k_j), written
    //      first and completed by the sparse part below
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

    // ---- sparse branch over the query blocks that selected J
    const int r0 = 16 * warp + (lane >> 2), r1 = r0 + 8;  // query rows of this thread's S fragments
    const int jm = 16 * (warp & 3), nh = 64 * (warp >> 2);  // key rows / column half of P^T dO, dS^T Q
    float dV[8][4], dK[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dV[n][e] = dK[n][e] = 0.0f;
    uint16_t *pt16 = reinterpret_cast<uint16_t *>(sm.pt), *dst16 = reinterpret_cast<uint16_t *>(sm.dst);
    const uint32_t *bits = selT + ((size_t)bh * n_kb + J) * n_awT;
    const int words = (n_qb + 31) / 32;
    for (int w = 0; w < words; ++w) {
        uint32_t b = __ldg(bits + w);
        while (b) {
            const int I = 32 * w + __ffs(b) - 1;
            b &= b - 1;
            const int i0 = I * blk_q, rows = min(blk_q, N - i0);
            __syncthreads();
            load_tile(sm.q, sm.qt, kRS, q + head, i0, rows, 128);
            load_tile(sm.dO, sm.dOt, kRS, dout + head, i0, rows, 128);
            if (tid < 128) {
                const bool ok = tid < rows;
                sm.m[tid] = ok ? __ldg(st_m + (size_t)bh * N + i0 + tid) : 0.0f;
                sm.l[tid] = ok ? __ldg(st_l + (size_t)bh * N + i0 + tid) : 0.0f;
                sm.D[tid] = ok ? __ldg(st_D + (size_t)bh * N + i0 + tid) : 0.0f;
            }
            __syncthreads();
            float s[8][4], dp[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.0f;
            warp_gemm<8>(s, sm.q, kRS, 16 * warp, sm.k, kRS, 0, 128);
            warp_gemm<8>(dp, sm.dO, kRS, 16 * warp, sm.v, kRS, 0, 128);
            const float mq0 = sm.m[r0], lq0 = sm.l[r0], Dq0 = sm.D[r0];
            const float mq1 = sm.m[r1], lq1 = sm.l[r1], Dq1 = sm.D[r1];
            const bool v0 = r0 < rows, v1 = r1 < rows;
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int j = 8 * n + 2 * tq + h;
                    const float p0 = (v0 && j < kv) ? __expf(s[n][h] * kRsd - mq0) * lq0 : 0.0f;
                    const float p1 = (v1 && j < kv) ? __expf(s[n][2 + h] * kRsd - mq1) * lq1 : 0.0f;
                    pt16[j * 2 * kRS + r0] = __bfloat16_as_ushort(__float2bfloat16_rn(p0));
                    pt16[j * 2 * kRS + r1] = __bfloat16_as_ushort(__float2bfloat16_rn(p1));
                    dst16[j * 2 * kRS + r0] = __bfloat16_as_ushort(__float2bfloat16_rn(p0 * (dp[n][h] - Dq0) * kRsd));
                    dst16[j * 2 * kRS + r1] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(p1 * (dp[n][2 + h] - Dq1) * kRsd));
                }
            __syncthreads();
            warp_gemm<8>(dV, sm.pt, kRS, jm, sm.dOt, kRS, nh, 128);  // dv += P^T dO
            warp_gemm<8>(dK, sm.dst, kRS, jm, sm.qt, kRS, nh, 128);  // dk += dS^T q / sqrt(d)
        }
    }
    __syncthreads();  // the linear part's dk, dv rows are written
    const int j0 = jm + (lane >> 2), j1 = j0 + 8;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
        const int c = nh + 8 * n + 2 * tq;
        if (j0 < kv) {
            float2 *pk = reinterpret_cast<float2 *>(dk + head + (size_t)(t0 + j0) * 128 + c);
            float2 *pv = reinterpret_cast<float2 *>(dv + head + (size_t)(t0 + j0) * 128 + c);
            const float2 ok_ = *pk, ov_ = *pv;
            *pk = make_float2(ok_.x + dK[n][0], ok_.y + dK[n][1]);
            *pv = make_float2(ov_.x + dV[n][0], ov_.y + dV[n][1]);
        }
        if (j1 < kv) {
            float2 *pk = reinterpret_cast<float2 *>(dk + head + (size_t)(t0 + j1) * 128 + c);
            float2 *pv = reinterpret_cast<float2 *>(dv + head + (size_t)(t0 + j1) * 128 + c);
            const float2 ok_ = *pk, ov_ = *pv;
            *pk = make_float2(ok_.x + dK[n][2], ok_.y + dK[n][3]);
            *pv = make_float2(ov_.x + dV[n][2], ov_.y + dV[n][3]);
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
    // 1. the forward's selection and states (quantisation off)
    BWD_TRY(launch_pool(q, g.BH, g.N, g.blk_q, g.n_qb, qbar, nullptr, s));
    BWD_TRY(launch_pool(k, g.BH, g.N, g.blk_k, g.n_kb, kbar, nullptr, s));
    BWD_TRY(launch_states(k, v, g, phi, states, partials, nullptr, status, s));
    BWD_TRY(launch_htot(partials, g, htot, s));
    BWD_TRY(launch_scores(qbar, kbar, g, scores, s));
    BWD_TRY(launch_topk(scores, g, idx, nullptr, amask, s));
    BWD_TRY(launch_state_reduce(amask, states, htot, g, hq, status, s));
    // 2. query side
    const int ks = g.k_sel;
    {
        const size_t smem = sizeof(QuerySmem) + 16;
        BWD_TRY(cudaFuncSetAttribute(bwd_query_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        bwd_query_kernel<<<dim3(g.n_qb, g.BH), kBwdThreads, smem, s>>>(
            static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(k), static_cast<const uint16_t *>(v),
            static_cast<const uint16_t *>(dout), idx, hq, g.N, g.blk_q, g.n_qb, ks, phi, dq, st_m, st_l, st_D, dh32,
            dh16);
        BWD_TRY(cudaGetLastError());
    }
    // 3. column sum of dH over the query blocks; transposed selection bits
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
    // 4. G = A^T dH (the state reduction on the transposed mask)
    {
        Geometry gt = g;
        gt.n_qb = g.n_kb;
        gt.n_kb = g.n_qb;
        gt.n_aw = L.n_awT;
        BWD_TRY(launch_state_reduce(amaskT, dh16, dhtot, gt, G, status, s));
    }
    // 5. key side
    {
        const size_t smem = sizeof(KeySmem) + 16;
        BWD_TRY(cudaFuncSetAttribute(bwd_key_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        bwd_key_kernel<<<dim3(g.n_kb, g.BH), kBwdThreads, smem, s>>>(
            static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(k), static_cast<const uint16_t *>(v),
            static_cast<const uint16_t *>(dout), selT, L.n_awT, G, st_m, st_l, st_D, g.N, g.blk_q, g.n_qb, g.n_kb,
            phi, dk, dv);
        BWD_TRY(cudaGetLastError());
    }
#undef BWD_TRY
    return cudaSuccess;
}

}  // namespace sla
