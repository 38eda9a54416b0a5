// sla_attention.cu -- fused block-sparse attention + linear epilogue of the
// SageSLA forward (one CTA per (batch*head, query block)).
//
// Sparse branch: exact softmax attention softmax(q k^T / sqrt(d)) v
// ("TurboDiffusion技术架构解析" §2.1, standard attention formula) over the tokens
// of the key blocks the query block selected, computed SageAttention-style
// ("清华开源TurboDiffusion加速框架", SageAttention与稀疏计算): INT8 Q.K^T on the
// tensor cores with per-block fp32 dequantisation scales, online softmax in
// fp32, P rounded to bf16 for a bf16 P.V with fp32 accumulation.  With
// quantisation off, Q.K^T runs in bf16 with fp32 accumulation.
//
// Linear branch epilogue: phi(Q_I) H_I as a tf32 MMA into its own TMEM
// accumulator, normalised by phi(q) . Z_I on the CUDA cores; output =
// sparse + linear, rounded to bf16.
//
// Roles (192 threads): warp 0 issues TMA loads, warp 1 issues tcgen05 MMAs and
// owns TMEM, warps 2-5 (one TMEM lane quarter each, one query row per thread)
// run softmax, the O correction and the epilogue.  Tensor memory columns:
// S double buffer [0,128), O [128,256), L [256,384).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sla_internal.h"
#include "sla_ptx.cuh"

namespace sla {
namespace {

constexpr int kAttnThreads = 192;
constexpr uint32_t kBox = 64 * 128;          // [64 rows x 128 B]
constexpr uint32_t kQRowsBox = 128 * 128;    // [128 rows x 128 B]
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;    // log2 units: P may grow to 2^8 before O is rescaled
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1 / sqrt(128)

template <bool QUANT>
struct AttnCfg {
    static constexpr uint32_t kQBytes = QUANT ? kQRowsBox : 2 * kQRowsBox;   // Q tile
    static constexpr uint32_t kKBytes = QUANT ? kBox : 2 * kBox;             // one key block of K
    static constexpr uint32_t kVBytes = 2 * kBox;                            // one key block of V
    static constexpr uint32_t kStageBytes = kKBytes + kVBytes;
    static constexpr int kStages = QUANT ? 5 : 4;
    static constexpr uint32_t kLinBytes = 8 * kQRowsBox;                     // phi(Q) 64 KB + H_I 64 KB
    static constexpr uint32_t kRegion = (kStages * kStageBytes > kLinBytes) ? kStages * kStageBytes : kLinBytes;
};

template <bool QUANT>
struct AttnSmem {
    alignas(1024) uint8_t q[AttnCfg<QUANT>::kQBytes];
    alignas(1024) uint8_t p[2][kQRowsBox];
    alignas(1024) uint8_t region[AttnCfg<QUANT>::kRegion];  // linear operands, then the K/V ring
    float z[kD];
    uint64_t bar_q, bar_h, bar_phiq, bar_lin, drain;
    uint64_t full[AttnCfg<QUANT>::kStages], empty[AttnCfg<QUANT>::kStages];
    uint64_t bar_s[2], bar_sfree[2], bar_p[2], bar_pv[2];
    uint32_t tmem_base;
    int abort_flag;
};

SLA_DEV float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

SLA_DEV float phi_f(float x, int phi)
{
    if (phi == 1) return fmaxf(x, 0.0f);
    return x > 0.0f ? x + 1.0f : expf(x);
}

SLA_DEV void named_bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

template <bool QUANT>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_h,
            const uint16_t *__restrict__ qraw, const float *__restrict__ qscale, const float *__restrict__ kscale,
            const int32_t *__restrict__ idx, const float *__restrict__ hq, int N, int blk_q, int n_qb, int n_kb,
            int k_sel, int phi, uint16_t *__restrict__ out, int *status)
{
    using Cfg = AttnCfg<QUANT>;
    constexpr int NS = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    AttnSmem<QUANT> &sm =
        *reinterpret_cast<AttnSmem<QUANT> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int I = blockIdx.x, bh = blockIdx.y;
    const int32_t *sel = idx + ((size_t)bh * n_qb + I) * k_sel;
    volatile int *abort_flag = &sm.abort_flag;
    if (tid == 0) sm.abort_flag = global_failed(status) ? 1 : 0;
    __syncthreads();
    if (sm.abort_flag) return;  // another CTA already failed: CTA-uniform early exit

    if (tid == 0) {
        mbar_init(&sm.bar_q, 1);
        mbar_init(&sm.bar_h, 1);
        mbar_init(&sm.bar_phiq, 128);
        mbar_init(&sm.bar_lin, 1);
        mbar_init(&sm.drain, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.bar_s[b], 1);
            mbar_init(&sm.bar_sfree[b], 128);
            mbar_init(&sm.bar_p[b], 128);
            mbar_init(&sm.bar_pv[b], 1);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t t_s = tmem, t_o = tmem + 128, t_l = tmem + 256;
    uint8_t *phiq_s = sm.region;                    // 4 x [128 rows x 32 fp32]
    uint8_t *h_s = sm.region + 4 * kQRowsBox;       // 4 x [128 dims x 32 fp32]

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_h);
            const int row0 = I * blk_q;
            mbar_expect_tx(&sm.bar_h, 4 * kQRowsBox);
            for (int c = 0; c < 4; ++c) tma_load_3d(h_s + c * kQRowsBox, &tm_h, &sm.bar_h, 32 * c, 0, bh * n_qb + I);
            if (k_sel > 0) {
                mbar_expect_tx(&sm.bar_q, Cfg::kQBytes);
                if (QUANT) {
                    tma_load_3d(sm.q, &tm_q, &sm.bar_q, 0, row0, bh);
                } else {
                    tma_load_3d(sm.q, &tm_q, &sm.bar_q, 0, row0, bh);
                    tma_load_3d(sm.q + kQRowsBox, &tm_q, &sm.bar_q, 64, row0, bh);
                }
            }
            int issued = 0;
            bool ok = mbar_wait(&sm.bar_lin, 0, status, abort_flag);  // region free of linear operands
            for (int j = 0; ok && j < k_sel; ++j) {
                const int s = j % NS, u = j / NS;
                if (u > 0 && !(ok = mbar_wait(&sm.empty[s], (u - 1) & 1, status, abort_flag))) break;
                const int J = __ldg(sel + j);
                uint8_t *st = sm.region + s * Cfg::kStageBytes;
                mbar_expect_tx(&sm.full[s], Cfg::kStageBytes);
                if (QUANT) {
                    tma_load_3d(st, &tm_k, &sm.full[s], 0, J * 64, bh);
                } else {
                    tma_load_3d(st, &tm_k, &sm.full[s], 0, J * 64, bh);
                    tma_load_3d(st + kBox, &tm_k, &sm.full[s], 64, J * 64, bh);
                }
                tma_load_3d(st + Cfg::kKBytes, &tm_v, &sm.full[s], 0, J * 64, bh);
                tma_load_3d(st + Cfg::kKBytes + kBox, &tm_v, &sm.full[s], 64, J * 64, bh);
                issued = j + 1;
            }
            if (!ok) {  // failure: let loads in flight land before shared memory is released
                mbar_wait_quiet(&sm.bar_h, 0);
                if (k_sel > 0) mbar_wait_quiet(&sm.bar_q, 0);
                for (int s = 0; s < NS; ++s) {
                    int jl = -1;
                    for (int j = s; j < issued; j += NS) jl = j;
                    if (jl >= 0) mbar_wait_quiet(&sm.full[s], (jl / NS) & 1);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = mbar_wait(&sm.bar_h, 0, status, abort_flag) && mbar_wait(&sm.bar_phiq, 0, status, abort_flag);
            if (ok) {
                tc_fence_after();
                constexpr uint32_t id_lin = idesc(1, 2, 2, 0, 0, 128, 128);  // f32 <- tf32 x tf32, K-major
                const uint32_t pa = smem_u32(phiq_s), ha = smem_u32(h_s);
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const uint32_t off = (k >> 2) * kQRowsBox + (k & 3) * 32;
                    mma_tf32(t_l, sdesc_sw128(pa + off, 16, 1024), sdesc_sw128(ha + off, 16, 1024), id_lin,
                             k > 0 ? 1u : 0u);
                }
                mma_commit(&sm.bar_lin);
            }
            constexpr uint32_t id_qk = QUANT ? idesc(2, 1, 1, 0, 0, 128, 64) : idesc(1, 1, 1, 0, 0, 128, 64);
            constexpr uint32_t id_pv = idesc(1, 1, 1, 0, 1, 128, 128);  // P K-major, V MN-major
            const uint32_t qa = smem_u32(sm.q);
            auto issue_qk = [&](int j) {
                const int s = j % NS, b = j & 1;
                const uint32_t ka = smem_u32(sm.region + s * Cfg::kStageBytes);
                if (QUANT) {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_i8(t_s + 64 * b, sdesc_sw128(qa + 32 * k, 16, 1024), sdesc_sw128(ka + 32 * k, 16, 1024),
                               id_qk, k > 0 ? 1u : 0u);
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16(t_s + 64 * b, sdesc_sw128(qa + (k >> 2) * kQRowsBox + 32 * (k & 3), 16, 1024),
                                 sdesc_sw128(ka + (k >> 2) * kBox + 32 * (k & 3), 16, 1024), id_qk, k > 0 ? 1u : 0u);
                }
                mma_commit(&sm.bar_s[b]);
            };
            if (ok && k_sel > 0) ok = mbar_wait(&sm.bar_q, 0, status, abort_flag);
            if (ok && k_sel > 0) ok = mbar_wait(&sm.full[0], 0, status, abort_flag);
            if (ok && k_sel > 0) {
                tc_fence_after();
                issue_qk(0);
            }
            for (int j = 0; ok && j < k_sel; ++j) {
                if (j + 1 < k_sel) {
                    const int jn = j + 1, b = jn & 1;
                    if (!(ok = mbar_wait(&sm.full[jn % NS], (jn / NS) & 1, status, abort_flag))) break;
                    if (jn >= 2 && !(ok = mbar_wait(&sm.bar_sfree[b], ((jn >> 1) - 1) & 1, status, abort_flag))) break;
                    tc_fence_after();
                    issue_qk(jn);
                }
                if (!(ok = mbar_wait(&sm.bar_p[j & 1], (j >> 1) & 1, status, abort_flag))) break;
                tc_fence_after();
                const uint32_t pa = smem_u32(sm.p[j & 1]);
                const uint32_t va = smem_u32(sm.region + (j % NS) * Cfg::kStageBytes + Cfg::kKBytes);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(t_o, sdesc_sw128(pa + 32 * k, 16, 1024), sdesc_sw128(va + 2048 * k, kBox, 1024), id_pv,
                             (j > 0 || k > 0) ? 1u : 0u);
                mma_commit(&sm.bar_pv[j & 1]);
                mma_commit(&sm.empty[j % NS]);
            }
            // every MMA retired before TMEM is released (normal and failure path)
            mma_commit(&sm.drain);
            mbar_wait_quiet(&sm.drain, 0);
        }
    } else {
        // ------------------------------------------------------------ softmax / epilogue
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;              // query row within the tile (= TMEM lane)
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int i = I * blk_q + r;
        const bool row_valid = r < blk_q && i < N;
        const int t128 = tid - 64;
        // Z_I into shared memory, then phi(q) -> tf32 -> phi(Q) tile, and den = phi(q).Z_I
        sm.z[t128] = __ldg(hq + ((size_t)bh * n_qb + I) * kStateCols + kD * kD + t128);
        named_bar_sync(1, 128);
        float den = 0.0f;
        {
            const uint4 *qr = reinterpret_cast<const uint4 *>(qraw + ((size_t)bh * N + (row_valid ? i : 0)) * kD);
#pragma unroll 4
            for (int u = 0; u < 16; ++u) {  // 8 channels per iteration
                uint4 w = row_valid ? __ldg(qr + u) : make_uint4(0, 0, 0, 0);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                float f[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    f[2 * e] = to_tf32(phi_f(__uint_as_float(ww[e] << 16), phi));
                    f[2 * e + 1] = to_tf32(phi_f(__uint_as_float(ww[e] & 0xFFFF0000u), phi));
                }
                if (!row_valid) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = 0.0f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) den = fmaf(f[e], sm.z[8 * u + e], den);
                // channels 8u..8u+7 = chunk (u/4), 16-byte units (2u)%8 and (2u+1)%8 of row r
                uint8_t *base = phiq_s + (u >> 2) * kQRowsBox;
                *reinterpret_cast<float4 *>(base + sw128_off(r, (2 * u) & 7)) = make_float4(f[0], f[1], f[2], f[3]);
                *reinterpret_cast<float4 *>(base + sw128_off(r, (2 * u + 1) & 7)) = make_float4(f[4], f[5], f[6], f[7]);
            }
        }
        fence_async_smem();
        mbar_arrive(&sm.bar_phiq);

        // ---- sparse loop
        const float sq = QUANT ? __ldg(qscale + (size_t)bh * n_qb + I) : 0.0f;
        const float kscale_log2 = kLog2e * kInvSqrtD;
        // every wait below is made warp-uniform so that warp-collective tcgen05
        // loads/stores and vote instructions are always reached by all lanes
        auto wait_all = [&](uint64_t *bar, uint32_t par) {
            const bool r = mbar_wait(bar, par, status, abort_flag);
            return __all_sync(0xffffffffu, r);
        };
        float m_used = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int j = 0; j < k_sel; ++j) {
            const int b = j & 1;
            if (!(ok = wait_all(&sm.bar_s[b], (j >> 1) & 1))) break;
            tc_fence_after();
            uint32_t s0[32], s1[32];
            tmem_ld32(t_s + 64 * b + lane_off, s0);
            tmem_ld32(t_s + 64 * b + 32 + lane_off, s1);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.bar_sfree[b]);
            const int J = __ldg(sel + j);
            const int valid = min(64, N - J * 64);
            // logits in log2 units: x_k * c (x_k = integer dot or fp32 dot)
            float c;
            float x[64];
            if (QUANT) {
                c = sq * __ldg(kscale + (size_t)bh * n_kb + J) * kscale_log2;
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    // exact int32 -> fp32 for |v| < 2^22 through the 1.5 * 2^23 bias
                    x[k] = __int_as_float((int)s0[k] + 0x4B400000) - 12582912.0f;
                    x[k + 32] = __int_as_float((int)s1[k] + 0x4B400000) - 12582912.0f;
                }
            } else {
                c = kscale_log2;
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    x[k] = __uint_as_float(s0[k]);
                    x[k + 32] = __uint_as_float(s1[k]);
                }
            }
            float xmax = -INFINITY;
#pragma unroll
            for (int k = 0; k < 64; ++k)
                if (k < valid) xmax = fmaxf(xmax, x[k]);
            const float tmax = xmax * c;  // c >= 0
            const float m_new = fmaxf(m_used, tmax);
            const bool need = m_new > m_used + kRescaleThreshold;
            float alpha = 1.0f;
            if (need) {
                alpha = ex2(m_used - m_new);  // 0 when m_used = -inf
                m_used = m_new;
                l *= alpha;
            }
            // P buffer b was last read by PV(j-2)
            if (j >= 2 && !(ok = wait_all(&sm.bar_pv[b], ((j >> 1) - 1) & 1))) break;
            // O correction (warp-uniform: tcgen05.ld/st are warp-collective)
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                if (!(ok = wait_all(&sm.bar_pv[(j - 1) & 1], ((j - 1) >> 1) & 1))) break;
                tc_fence_after();
#pragma unroll 1
                for (int c0 = 0; c0 < kD; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(t_o + c0 + lane_off, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(t_o + c0 + lane_off, o);
                }
                tmem_wait_st();
            }
            const float neg_m = -m_used;
            float rs = 0.0f;
            uint8_t *prow = sm.p[b];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                float pv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int k = 8 * u + e;
                    pv[e] = (k < valid) ? ex2(fmaf(x[k], c, neg_m)) : 0.0f;
                    rs += pv[e];
                }
                *reinterpret_cast<uint4 *>(prow + sw128_off(r, u)) =
                    make_uint4(pack_bf16x2(pv[0], pv[1]), pack_bf16x2(pv[2], pv[3]), pack_bf16x2(pv[4], pv[5]),
                               pack_bf16x2(pv[6], pv[7]));
            }
            l += rs;
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&sm.bar_p[b]);
        }
        // ---- epilogue: out = O / l + L / den
        if (ok && k_sel > 0) ok = wait_all(&sm.bar_pv[(k_sel - 1) & 1], ((k_sel - 1) >> 1) & 1);
        if (ok) ok = wait_all(&sm.bar_lin, 0);
        if (ok) {
            tc_fence_after();
            const float inv_l = (k_sel > 0 && l > 0.0f) ? 1.0f / l : 0.0f;
            const float inv_den = den != 0.0f ? 1.0f / den : 0.0f;
            uint16_t *orow = out + ((size_t)bh * N + (row_valid ? i : 0)) * kD;
#pragma unroll 1
            for (int c0 = 0; c0 < kD; c0 += 32) {
                uint32_t lr[32], orr[32];
                tmem_ld32(t_l + c0 + lane_off, lr);
                if (k_sel > 0) tmem_ld32(t_o + c0 + lane_off, orr);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float a0 = __uint_as_float(lr[2 * e]) * inv_den, a1 = __uint_as_float(lr[2 * e + 1]) * inv_den;
                    if (k_sel > 0) {
                        a0 = fmaf(__uint_as_float(orr[2 * e]), inv_l, a0);
                        a1 = fmaf(__uint_as_float(orr[2 * e + 1]), inv_l, a1);
                    }
                    pk[e] = pack_bf16x2(a0, a1);
                }
                if (row_valid) {
                    uint4 *o4 = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
                    for (int e = 0; e < 4; ++e) o4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    __syncwarp();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <bool QUANT>
cudaError_t launch_attn_t(const void *q, const void *k, const void *v, const int8_t *q8, const int8_t *k8,
                          const float *qscale, const float *kscale, const int32_t *idx, const float *hq,
                          const Geometry &g, int phi, void *out, int *status, cudaStream_t s)
{
    CUtensorMap tq, tk, tv, th;
    const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)g.N, (uint64_t)g.BH};
    if (QUANT) {
        const uint64_t st[2] = {(uint64_t)kD, (uint64_t)g.N * kD};
        const uint32_t bq[3] = {128, 128, 1}, bk[3] = {128, 64, 1};
        if (!encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q8, dims, st, bq)) return cudaErrorInvalidValue;
        if (!encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, k8, dims, st, bk)) return cudaErrorInvalidValue;
    } else {
        const uint64_t st[2] = {(uint64_t)kD * 2, (uint64_t)g.N * kD * 2};
        const uint32_t bq[3] = {64, 128, 1}, bk[3] = {64, 64, 1};
        if (!encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, dims, st, bq)) return cudaErrorInvalidValue;
        if (!encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dims, st, bk)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t st[2] = {(uint64_t)kD * 2, (uint64_t)g.N * kD * 2};
        const uint32_t bv[3] = {64, 64, 1};
        if (!encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dims, st, bv)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t hd[3] = {(uint64_t)kD, (uint64_t)kD, (uint64_t)g.BH * g.n_qb};
        const uint64_t st[2] = {(uint64_t)kD * 4, (uint64_t)kStateCols * 4};
        const uint32_t bh[3] = {32, 128, 1};
        if (!encode_tmap(&th, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, hq, hd, st, bh)) return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(AttnSmem<QUANT>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<QUANT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(g.n_qb, g.BH);
    attn_kernel<QUANT><<<grid, kAttnThreads, smem, s>>>(tq, tk, tv, th, static_cast<const uint16_t *>(q), qscale, kscale,
                                                        idx, hq, g.N, g.blk_q, g.n_qb, g.n_kb, g.k_sel, phi,
                                                        static_cast<uint16_t *>(out), status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const void *q, const void *k, const void *v, const int8_t *q8, const int8_t *k8,
                             const float *qscale, const float *kscale, const int32_t *idx, const float *hq,
                             const Geometry &g, int phi, void *out, int *status, cudaStream_t s)
{
    if (g.quant) return launch_attn_t<true>(q, k, v, q8, k8, qscale, kscale, idx, hq, g, phi, out, status, s);
    return launch_attn_t<false>(q, k, v, q8, k8, qscale, kscale, idx, hq, g, phi, out, status, s);
}

}  // namespace sla
