// sla_w8a8.cu -- W8A8 INT8 linear layer with FusedNorm on tcgen05 tensor cores.
//
// "清华开源TurboDiffusion加速框架" (W8A8 INT8量化) and "TurboDiffusion：让可视化视频
// 生成效率提升200倍的加速引擎" (§1): the linear layers' weights and activations
// are quantised to 8-bit integers and run on the INT8 units, with a FusedNorm
// operator.  The
// granularity, rounding and norm are not stated; what is implemented:
//
//  rowquant_kernel  per row of a bf16 matrix [rows, cols]: optionally the RMS
//                   normalisation y = fp32(x * r) * gamma[c] with ms = (fp64 sum
//                   of x^2) / cols rounded to fp32 and r = 1 / sqrt(ms + eps)
//                   (IEEE fp32 add, sqrt, divide) -- the FusedNorm reading --
//                   then one symmetric INT8 scale per row, scale = amax / 127,
//                   code = clamp(rint_even(y / scale), +-127).  Activations take
//                   one scale per token, weights one per output channel.
//  w8a8_gemm_kernel out[m][n] = bf16( float(sum_k qx[m][k] qw[n][k]) * sx[m] *
//                   sw[n] + bias[n] ): a persistent tcgen05 kind::i8 GEMM (M =
//                   128 tokens x N = 256 channels per tile, int32 accumulators
//                   double-buffered in TMEM so one tile's epilogue overlaps the
//                   next tile's MMAs), K-major operands through a 4-stage TMA ring.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "sla_internal.h"
#include "sla_ptx.cuh"

namespace sla {
namespace {

// ---------------------------------------------------------------------------
// per-row quantisation (+ FusedNorm)
// ---------------------------------------------------------------------------
constexpr int kRqThreads = 256;
constexpr int kRqMaxChunks = 8;  // uint4 (8 bf16) per thread: cols <= 256 * 8 * 8 = 16384

// kRqChunks: uint4 per thread, the smallest instantiation that holds the row, so that
// short rows keep few registers and many CTAs (rows) in flight per SM
template <bool NORM, int kRqChunks>
__global__ void __launch_bounds__(kRqThreads) rowquant_kernel(const uint4 *__restrict__ x, int cols,
                                                              const float *__restrict__ gamma, float eps,
                                                              uint2 *__restrict__ q, float *__restrict__ scale)
{
    __shared__ double red_d[kRqThreads / 32];
    __shared__ float red_f[kRqThreads / 32];
    const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nch = cols / 8;  // 16-byte chunks in the row
    const uint4 *xr = x + (size_t)row * nch;
    uint4 raw[kRqChunks];
#pragma unroll
    for (int l = 0; l < kRqChunks; ++l) {
        const int e = tid + kRqThreads * l;
        raw[l] = e < nch ? __ldg(xr + e) : make_uint4(0, 0, 0, 0);
    }
    auto expand = [](const uint4 &u, float (&f)[8]) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    };
    float r = 1.0f;
    if (NORM) {
        // sum of squares in fp64 (a bf16 square is exact in fp64)
        double ss = 0.0;
#pragma unroll
        for (int l = 0; l < kRqChunks; ++l) {
            float f[8];
            expand(raw[l], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) ss = fma((double)f[i], (double)f[i], ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) red_d[warp] = ss;
        __syncthreads();
        double tot = 0.0;
#pragma unroll
        for (int w = 0; w < kRqThreads / 32; ++w) tot += red_d[w];
        const float ms = (float)(tot / (double)cols);
        r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    }
    // y and its row amax (y recomputed in the code pass)
    auto norm_chunk = [&](int l, float (&f)[8]) {
        expand(raw[l], f);
        if (NORM) {
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(f[i], r);
            if (gamma) {  // 8 consecutive channels: two 16-byte loads (gamma is 16-byte aligned)
                const float4 *g4 = reinterpret_cast<const float4 *>(gamma) + 2 * (tid + kRqThreads * l);
                const float4 ga = __ldg(g4), gb = __ldg(g4 + 1);
                const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(f[i], gg[i]);
            }
        }
    };
    float amax = 0.0f;
#pragma unroll
    for (int l = 0; l < kRqChunks; ++l) {
        if (tid + kRqThreads * l < nch) {
            float f[8];
            norm_chunk(l, f);
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) red_f[warp] = amax;
    __syncthreads();
    amax = red_f[0];
#pragma unroll
    for (int w = 1; w < kRqThreads / 32; ++w) amax = fmaxf(amax, red_f[w]);
    const float s = __fdiv_rn(amax, 127.0f);
    if (tid == 0) scale[row] = s;
    // codes: the reciprocal-product screen of the attention quantisation (rint(t) is the code
    // unless t = y * fl(1/s) lies within 2^-14 of a half-integer; then the IEEE quotient)
    const float rs = s != 0.0f ? __fdiv_rn(1.0f, s) : 0.0f;
    const bool fast = s != 0.0f && isfinite(rs);
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    uint2 *qr = q + (size_t)row * nch;
#pragma unroll
    for (int l = 0; l < kRqChunks; ++l) {
        const int e = tid + kRqThreads * l;
        if (e < nch) {
            float f[8];
            norm_chunk(l, f);
            uint32_t cb[8];
            unsigned slow = fast ? 0u : 0xFFu;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float t = f[i] * rs;
                const float qf = __fadd_rn(t, kRound);
                const float rt = __fsub_rn(qf, kRound);
                if (fabsf(t - rt) > 0.5f - 6.103515625e-05f) slow |= 1u << i;
                cb[i] = __float_as_uint(qf);
            }
            if (slow) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (slow & (1u << i))
                        cb[i] = s != 0.0f ? (uint32_t)max(-127, min(127, __float2int_rn(__fdiv_rn(f[i], s)))) : 0u;
            }
            const uint32_t w0 = __byte_perm(__byte_perm(cb[0], cb[1], 0x0040), __byte_perm(cb[2], cb[3], 0x0040), 0x5410);
            const uint32_t w1 = __byte_perm(__byte_perm(cb[4], cb[5], 0x0040), __byte_perm(cb[6], cb[7], 0x0040), 0x5410);
            qr[e] = make_uint2(w0, w1);
        }
    }
}

// ---------------------------------------------------------------------------
// W8A8 GEMM: warp 0 TMA producer, warp 1 MMA issuer (TMEM owner), warps 2..5
// epilogue (TMEM lane quarter = warp index % 4)
// ---------------------------------------------------------------------------
constexpr int kGmThreads = 192;
constexpr int kGmStages = 4;
constexpr int kGmBM = 128, kGmBN = 256, kGmBK = 128;  // BK in bytes = int8 elements
constexpr uint32_t kGmA = kGmBM * kGmBK;             // 16 KB
constexpr uint32_t kGmB = kGmBN * kGmBK;             // 32 KB

struct GemmSmem {
    alignas(1024) uint8_t a[kGmStages][kGmA];
    alignas(1024) uint8_t b[kGmStages][kGmB];
    uint64_t full[kGmStages], empty[kGmStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

__global__ void __launch_bounds__(kGmThreads, 1) w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                                  const __grid_constant__ CUtensorMap tm_w, int M,
                                                                  int N, int K, const float *__restrict__ sx,
                                                                  const float *__restrict__ sw,
                                                                  const float *__restrict__ bias,
                                                                  __nv_bfloat16 *__restrict__ out, int *status)
{
    extern __shared__ uint8_t smem_raw[];
    GemmSmem &sm = *reinterpret_cast<GemmSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_nt = (N + kGmBN - 1) / kGmBN, n_mt = (M + kGmBM - 1) / kGmBM;
    const int n_tiles = n_mt * n_nt, nk = (K + kGmBK - 1) / kGmBK;
    volatile int *abort_flag = &sm.abort_flag;
    if (tid == 0) sm.abort_flag = global_failed(status) ? 1 : 0;
    __syncthreads();
    if (sm.abort_flag) return;  // another CTA already failed: CTA-uniform early exit

    if (tid == 0) {
        for (int s = 0; s < kGmStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 128);
        }
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // tile t: n fastest, so the tiles that share one activation tile run together (weights stay in L2)
    auto tile_coords = [&](int t, int &m0, int &n0) {
        m0 = (t / n_nt) * kGmBM;
        n0 = (t % n_nt) * kGmBN;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int kc = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
            int m0, n0;
            tile_coords(t, m0, n0);
            for (int kt = 0; kt < nk; ++kt, ++kc) {
                const int s = kc % kGmStages, u = kc / kGmStages;
                if (u > 0 && !(ok = mbar_wait_warp(&sm.empty[s], (u - 1) & 1, status, abort_flag))) break;
                if (elect_one()) {
                    mbar_expect_tx(&sm.full[s], kGmA + kGmB);
                    tma_load_2d(sm.a[s], &tm_x, &sm.full[s], kt * kGmBK, m0);
                    tma_load_2d(sm.b[s], &tm_w, &sm.full[s], kt * kGmBK, n0);
                }
                __syncwarp();
            }
        }
        if (!ok && elect_one()) {  // loads in flight land before the CTA exits
            for (int s = 0; s < kGmStages; ++s) {
                int jl = -1;
                for (int j = s; j < kc; j += kGmStages) jl = j;
                if (jl >= 0) mbar_wait_quiet(&sm.full[s], (jl / kGmStages) & 1, status);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t kId = idesc(2, 1, 1, 0, 0, kGmBM, kGmBN);  // S32 <- s8 x s8, both K-major
        const uint64_t ad0 = sdesc_sw128(smem_u32(sm.a[0]), 16, 1024);
        const uint64_t bd0 = sdesc_sw128(smem_u32(sm.b[0]), 16, 1024);
        int kc = 0, lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++lt) {
            const int buf = lt & 1;
            const uint32_t acc = tmem + 256 * buf;
            if (lt >= 2 && !(ok = mbar_wait_warp(&sm.acc_empty[buf], ((lt >> 1) - 1) & 1, status, abort_flag))) break;
            tc_fence_after();
            for (int kt = 0; kt < nk; ++kt, ++kc) {
                const int s = kc % kGmStages, u = kc / kGmStages;
                if (!(ok = mbar_wait_warp(&sm.full[s], u & 1, status, abort_flag))) break;
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int k = 0; k < 4; ++k)  // K-step of 32 int8 = 32 bytes
                        mma_i8(acc, ad0 + (uint64_t)((s * kGmA + 32 * k) >> 4), bd0 + (uint64_t)((s * kGmB + 32 * k) >> 4),
                               kId, (kt > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&sm.empty[s]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (elect_one()) mma_commit(&sm.acc_full[buf]);
            __syncwarp();
        }
        if (elect_one()) {
            mma_commit(&sm.drain);
            mbar_wait_quiet(&sm.drain, 0, status);  // MMAs retired before TMEM is freed
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        int lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++lt) {
            int m0, n0;
            tile_coords(t, m0, n0);
            const int buf = lt & 1;
            if (!(ok = mbar_wait_warp(&sm.acc_full[buf], (lt >> 1) & 1, status, abort_flag))) break;
            tc_fence_after();
            const int m = m0 + 32 * q + lane;
            const float sxm = m < M ? __ldg(sx + m) : 0.0f;
            __nv_bfloat16 *orow = out + (size_t)(m < M ? m : 0) * N;
#pragma unroll 1
            for (int c0 = 0; c0 < kGmBN; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(tmem + 256 * buf + ((uint32_t)(32 * q) << 16) + c0, r);
                tmem_wait_ld();
                const int n = n0 + c0;
                if (m < M && n < N) {  // N % 8 == 0: whole 8-column groups are in range or out
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float v[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int nn = min(n + 2 * i + h, N - 1);
                            float y = (float)(int)r[2 * i + h] * sxm * __ldg(sw + nn);
                            if (bias) y += __ldg(bias + nn);
                            v[h] = y;
                        }
                        pk[i] = pack_bf16x2(v[0], v[1]);
                    }
                    uint4 *o4 = reinterpret_cast<uint4 *>(orow + n);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (n + 8 * i < N) o4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.acc_empty[buf]);
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

}  // namespace

cudaError_t launch_rowquant(const void *x, int rows, int cols, int norm, const float *gamma, float eps, int8_t *q,
                            float *scale, cudaStream_t s)
{
    if (cols % 8 != 0 || cols > kRqThreads * kRqMaxChunks * 8) return cudaErrorInvalidValue;
    const uint4 *xi = static_cast<const uint4 *>(x);
    uint2 *qo = reinterpret_cast<uint2 *>(q);
    const int ch = (cols / 8 + kRqThreads - 1) / kRqThreads;
    auto go = [&](auto chunks) {
        constexpr int C = decltype(chunks)::value;
        if (norm) rowquant_kernel<true, C><<<rows, kRqThreads, 0, s>>>(xi, cols, gamma, eps, qo, scale);
        else rowquant_kernel<false, C><<<rows, kRqThreads, 0, s>>>(xi, cols, nullptr, 0.0f, qo, scale);
    };
    if (ch <= 1) go(std::integral_constant<int, 1>{});
    else if (ch <= 2) go(std::integral_constant<int, 2>{});
    else if (ch <= 3) go(std::integral_constant<int, 3>{});
    else if (ch <= 4) go(std::integral_constant<int, 4>{});
    else go(std::integral_constant<int, 8>{});
    return cudaGetLastError();
}

cudaError_t launch_w8a8_gemm(const int8_t *qx, const float *sx, const int8_t *qw, const float *sw, const float *bias,
                             int M, int N, int K, void *out, int *status, cudaStream_t s)
{
    CUtensorMap tx, tw;
    {
        const uint64_t dims[2] = {(uint64_t)K, (uint64_t)M};
        const uint64_t strides[1] = {(uint64_t)K};
        const uint32_t box[2] = {(uint32_t)kGmBK, (uint32_t)kGmBM};
        if (!encode_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, qx, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[2] = {(uint64_t)K, (uint64_t)N};
        const uint64_t strides[1] = {(uint64_t)K};
        const uint32_t box[2] = {(uint32_t)kGmBK, (uint32_t)kGmBN};
        if (!encode_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, qw, dims, strides, box)) return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(GemmSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(w8a8_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_tiles = ((M + kGmBM - 1) / kGmBM) * ((N + kGmBN - 1) / kGmBN);
    w8a8_gemm_kernel<<<n_tiles < sms ? n_tiles : sms, kGmThreads, smem, s>>>(
        tx, tw, M, N, K, sx, sw, bias, static_cast<__nv_bfloat16 *>(out), status);
    return cudaGetLastError();
}

}  // namespace sla

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
#include "../../include/sla.h"

namespace {
bool al(const void *p, uintptr_t a) { return p != nullptr && ((uintptr_t)p & (a - 1)) == 0; }
}  // namespace

namespace sla {
cudaError_t set_wait_budget_w8a8(long long cycles) { return set_tu_wait_budget(cycles); }
}  // namespace sla

extern "C" {

size_t sla_w8a8_workspace_bytes(void) { return 256; }

sla_status sla_w8a8_quantize(const void *x, int rows, int cols, int norm, const float *gamma, float eps, int8_t *q,
                             float *scale, void *stream)
{
    if (rows < 1 || cols < 8 || (norm != 0 && norm != 1)) return SLA_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !(eps < 1e30f)) return SLA_ERR_INVALID_ARG;
    if (cols % 8 != 0 || cols > 16384) return SLA_ERR_UNSUPPORTED;
    if (!al(x, 16) || !al(q, 16) || !al(scale, 4) || (gamma && !al(gamma, 16))) return SLA_ERR_INVALID_ARG;
    if (sla::launch_rowquant(x, rows, cols, norm, norm ? gamma : nullptr, eps, q, scale,
                             static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return SLA_ERR_CUDA;
    return SLA_OK;
}

sla_status sla_w8a8_linear(const int8_t *qx, const float *sx, const int8_t *qw, const float *sw, const float *bias,
                           int M, int N, int K, void *out, void *ws, size_t ws_bytes, void *stream)
{
    if (M < 1 || N < 1 || K < 1) return SLA_ERR_INVALID_ARG;
    if (K % 16 != 0 || N % 8 != 0) return SLA_ERR_UNSUPPORTED;
    if (!al(qx, 16) || !al(qw, 16) || !al(out, 16) || !al(ws, 16) || !al(sx, 4) || !al(sw, 4) ||
        (bias && !al(bias, 4)))
        return SLA_ERR_INVALID_ARG;
    if (ws_bytes < sla_w8a8_workspace_bytes()) return SLA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int *status = static_cast<int *>(ws);
    if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return SLA_ERR_CUDA;
    if (sla::launch_w8a8_gemm(qx, sx, qw, sw, bias, M, N, K, out, status, s) != cudaSuccess) return SLA_ERR_CUDA;
    return SLA_OK;
}

}  // extern "C"
