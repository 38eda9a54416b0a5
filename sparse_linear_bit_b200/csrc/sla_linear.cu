// sla_linear.cu -- linear branch of the SageSLA forward on tcgen05 tensor cores.
//
// Kernelised linear attention phi(Q)(phi(K)^T V) ("TurboDiffusion技术架构解析"
// §2.1, phi = elu+1 or ReLU) applied, for query block I, to the key blocks I
// did not select.  Three kernels:
//
//  states_kernel  per key block J: hT_J = V_J^T phi(K_J) (128 x 128, fp16 MMA:
//                 phi(K) and V converted to fp16 in shared memory, saturating
//                 at +-65504; fp32 TMEM accumulator) stored bf16 as
//                 [dim][channel], and z_J = column sums of phi(K_J); a second
//                 accumulator sums the fp32 states of a chunk of 32 key blocks
//                 for the global state.  Optionally writes the fp16 copy of V
//                 that the attention kernel's fp16 P.V uses when quantisation
//                 is off.
//  htot_kernel    global state per head = fixed-order sum of the chunk sums.
//  reduce_kernel  per query block I: C_I = sum_J A[I][J] S_J as a dense GEMM
//                 (M = 128 query blocks, N = 256 state columns, K = key
//                 blocks) with a 0/1 mask A.  When at most half the key blocks
//                 are selected A marks the selected blocks and the state is
//                 H_total - C_I (only the selected ~10% go through bf16); else A
//                 marks the unselected blocks and the state is C_I (exact zeros
//                 when everything is selected).  Output fp32, the d x d part
//                 rounded to tf32 for the epilogue MMA of the attention kernel.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sla_internal.h"
#include "sla_ptx.cuh"

namespace sla {
namespace {

constexpr int kStatesThreads = 128;
constexpr uint32_t kTileBytes = 64 * 128;  // one [64 rows x 128 B] TMA box

struct StatesSmem {
    alignas(1024) uint8_t k[2][2][kTileBytes];  // [stage][channel half][64 tokens x 64 ch]
    alignas(1024) uint8_t v[2][2][kTileBytes];  // [stage][dim half][64 tokens x 64 dims]
    uint64_t full[2];
    uint64_t mma_done;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ float phi_f(float x, int phi)
{
    if (phi == 1) return fmaxf(x, 0.0f);
    return x > 0.0f ? x + 1.0f : expf(x);
}

__global__ void __launch_bounds__(kStatesThreads) states_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                                const __grid_constant__ CUtensorMap tm_v, int N,
                                                                int n_kb, int n_chunks, int phi,
                                                                uint16_t *__restrict__ states,
                                                                float *__restrict__ partials,
                                                                uint16_t *__restrict__ v16, int *status)
{
    extern __shared__ uint8_t smem_raw[];
    StatesSmem &sm = *reinterpret_cast<StatesSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = blockIdx.y, chunk = blockIdx.x;
    const int Jbeg = chunk * kStateChunk, nJ = min(kStateChunk, n_kb - Jbeg);
    volatile int *abort_flag = &sm.abort_flag;
    if (tid == 0) sm.abort_flag = global_failed(status) ? 1 : 0;
    __syncthreads();
    if (sm.abort_flag) return;  // another CTA already failed: CTA-uniform early exit

    if (tid == 0) {
        mbar_init(&sm.full[0], 1);
        mbar_init(&sm.full[1], 1);
        mbar_init(&sm.mma_done, 1);
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t d_blk = tmem, d_sum = tmem + 128;
    constexpr uint32_t kIdesc = idesc(1, 0, 0, 1, 1, 128, 128);  // f32 <- f16 (MN) x f16 (MN)

    auto issue = [&](int j) {
        const int s = j & 1, J = Jbeg + j;
        mbar_expect_tx(&sm.full[s], 4 * kTileBytes);
        tma_load_3d(sm.k[s][0], &tm_k, &sm.full[s], 0, J * 64, bh);
        tma_load_3d(sm.k[s][1], &tm_k, &sm.full[s], 64, J * 64, bh);
        tma_load_3d(sm.v[s][0], &tm_v, &sm.full[s], 0, J * 64, bh);
        tma_load_3d(sm.v[s][1], &tm_v, &sm.full[s], 64, J * 64, bh);
    };
    int issued = 0;
    if (tid == 0) {
        for (; issued < min(2, nJ); ++issued) issue(issued);
    }

    float zsum = 0.0f;
    bool ok = true;
    for (int j = 0; j < nJ && ok; ++j) {
        const int s = j & 1, J = Jbeg + j;
        ok = __syncthreads_and(mbar_wait(&sm.full[s], (j >> 1) & 1, status, abort_flag));
        if (!ok) break;
        // phi(K) and V to fp16 in place (elementwise, so the swizzle permutation
        // is irrelevant); tokens past N contribute nothing
        const int valid = min(64, N - J * 64);
#pragma unroll 2
        for (int l = 0; l < 16; ++l) {
            const int e = tid + kStatesThreads * l;  // 16-byte chunk 0..2047: K halves, then V halves
            const bool is_v = e >= 1024;
            const int e2 = e & 1023, half = e2 >> 9, row = (e2 & 511) >> 3;
            uint8_t *tile = is_v ? sm.v[s][half] : sm.k[s][half];
            uint4 *p = reinterpret_cast<uint4 *>(tile + (e2 & 511) * 16);
            uint4 w = *p;
            uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float a = __uint_as_float(ww[i] << 16), b = __uint_as_float(ww[i] & 0xFFFF0000u);
                if (!is_v) {
                    a = phi_f(a, phi);
                    b = phi_f(b, phi);
                }
                ww[i] = row < valid ? pack_f16x2_sat(a, b) : 0u;
            }
            *p = make_uint4(ww[0], ww[1], ww[2], ww[3]);
            if (is_v && v16 != nullptr && row < valid) {
                // un-swizzled fp16 copy of V: chunk (e2 & 7) of this row holds logical chunk ^ (row & 7)
                const int u = (e2 & 7) ^ (row & 7);
                *reinterpret_cast<uint4 *>(v16 + (((size_t)bh * N + J * 64 + row) * kD + half * 64 + u * 8)) =
                    make_uint4(ww[0], ww[1], ww[2], ww[3]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t ka = smem_u32(sm.k[s][0]), va = smem_u32(sm.v[s][0]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t ad = sdesc_sw128(va + 2048 * k, kTileBytes, 1024);  // A = V^T (dims x tokens)
                const uint64_t bd = sdesc_sw128(ka + 2048 * k, kTileBytes, 1024);  // B = phi(K) (ch x tokens)
                mma_bf16(d_blk, ad, bd, kIdesc, k > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t ad = sdesc_sw128(va + 2048 * k, kTileBytes, 1024);
                const uint64_t bd = sdesc_sw128(ka + 2048 * k, kTileBytes, 1024);
                mma_bf16(d_sum, ad, bd, kIdesc, (j > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit(&sm.mma_done);
        }
        // z_J[c] = sum over tokens of phi(K)[t][c] (thread = channel), row order
        {
            const int c = tid, half = c >> 6, u = (c & 63) >> 3, el = c & 7;
            const uint8_t *base = sm.k[s][half];
            float z = 0.0f;
            for (int r = 0; r < 64; ++r) {
                const __half b = *reinterpret_cast<const __half *>(base + sw128_off(r, u) + el * 2);
                z += __half2float(b);
            }
            zsum += z;
            const __nv_bfloat16 zb = __float2bfloat16_rn(z);
            states[((size_t)bh * n_kb + J) * kStateCols + kD * kD + c] = *reinterpret_cast<const uint16_t *>(&zb);
        }
        ok = __syncthreads_and(mbar_wait(&sm.mma_done, j & 1, status, abort_flag));
        if (!ok) break;
        tc_fence_after();
        // epilogue: thread = dim row d of hT_J (TMEM lane), 128 channel columns
        {
            const int d = tid;
            uint16_t *dst = states + ((size_t)bh * n_kb + J) * kStateCols + (size_t)d * kD;
#pragma unroll 1
            for (int c0 = 0; c0 < kD; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(d_blk + ((uint32_t)(warp * 32) << 16) + c0, r);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                uint4 *o = reinterpret_cast<uint4 *>(dst + c0);
#pragma unroll
                for (int i = 0; i < 4; ++i) o[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && issued < nJ) issue(issued++);
    }
    // chunk sum of the fp32 states
    if (ok && nJ > 0) {
        const int d = tid;
        float *dst = partials + ((size_t)bh * n_chunks + chunk) * kStateCols;
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(d_sum + ((uint32_t)(warp * 32) << 16) + c0, r);
            tmem_wait_ld();
            float4 *o = reinterpret_cast<float4 *>(dst + (size_t)d * kD + c0);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                o[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                   __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
        }
        dst[kD * kD + tid] = zsum;
    }
    if (!ok && tid == 0) {
        // drain: loads and MMAs still in flight retire before shared memory / TMEM are released
        for (int s = 0; s < 2; ++s) {
            const int jl = issued - 1 - ((issued - 1 - s) & 1);  // last load issued on stage s
            if (jl >= 0) mbar_wait_quiet(&sm.full[s], (jl >> 1) & 1);
        }
        mma_commit(&sm.drain);
        mbar_wait_quiet(&sm.drain, 0);
    }
    tc_fence_before();
    __syncthreads();
    __syncwarp();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// htot[bh][n] = sum over chunks (in order) of partials[bh][chunk][n]
__global__ void htot_kernel(const float *__restrict__ partials, int n_chunks, float *__restrict__ htot)
{
    const int bh = blockIdx.y, n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= kStateCols) return;
    const float *p = partials + (size_t)bh * n_chunks * kStateCols + n;
    float s = 0.0f;
    for (int c = 0; c < n_chunks; ++c) s += p[(size_t)c * kStateCols];
    htot[(size_t)bh * kStateCols + n] = s;
}

// ---------------------------------------------------------------------------
// per-query-block state: persistent GEMM over tiles (bh, 256 state columns,
// 128 query blocks), m fastest so the 5 query-block tiles of one column tile
// run together and share the state columns through L2.  Warp 0 = TMA producer,
// warp 1 = MMA issuer, warps 2..5 = epilogue (TMEM lanes by warp index % 4).
// Two TMEM accumulators: the epilogue of one tile overlaps the next tile's MMAs.
// ---------------------------------------------------------------------------
constexpr int kRedStages = 4;
constexpr int kRedThreads = 192;
constexpr uint32_t kRedA = 128 * 128;      // 128 query blocks x 64 key blocks (bf16)
constexpr uint32_t kRedB = 4 * kTileBytes; // 64 key blocks x 256 columns (bf16), four 64-column boxes

struct ReduceSmem {
    alignas(1024) uint8_t a[kRedStages][kRedA];
    alignas(1024) uint8_t b[kRedStages][kRedB];
    float ht[4][256];  // global-state columns of the tile in the epilogue, one copy per epilogue warp
    uint64_t full[kRedStages];
    uint64_t empty[kRedStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ uint64_t dadd16(uint64_t desc, uint32_t bytes) { return desc + (uint64_t)(bytes >> 4); }

__global__ void __launch_bounds__(kRedThreads, 1) reduce_kernel(const __grid_constant__ CUtensorMap tm_a,
                                                                const __grid_constant__ CUtensorMap tm_s, int n_qb,
                                                                int n_kb, int n_tiles, int subtract,
                                                                const float *__restrict__ htot,
                                                                float *__restrict__ hq, int *status)
{
    extern __shared__ uint8_t smem_raw[];
    ReduceSmem &sm = *reinterpret_cast<ReduceSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_mt = (n_qb + 127) / 128, n_nt = (kStateCols + 255) / 256;
    const int nk = (n_kb + 63) / 64;
    volatile int *abort_flag = &sm.abort_flag;
    if (tid == 0) sm.abort_flag = global_failed(status) ? 1 : 0;
    __syncthreads();
    if (sm.abort_flag) return;  // another CTA already failed: CTA-uniform early exit

    if (tid == 0) {
        for (int s = 0; s < kRedStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 128);
        }
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_s);
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    auto tile_coords = [&](int t, int &bh, int &I0, int &n0) {
        const int m = t % n_mt, rest = t / n_mt;
        bh = rest / n_nt;
        n0 = (rest % n_nt) * 256;
        I0 = m * 128;
    };

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ producer
        int kc = 0;  // k-steps issued over all tiles of this CTA
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
            int bh, I0, n0;
            tile_coords(t, bh, I0, n0);
            const int n_groups = min(256, kStateCols - n0) / 64;
            for (int kt = 0; kt < nk; ++kt, ++kc) {
                const int s = kc % kRedStages, u = kc / kRedStages;
                if (u > 0 && !(ok = mbar_wait(&sm.empty[s], (u - 1) & 1, status, abort_flag))) break;
                mbar_expect_tx(&sm.full[s], kRedA + (uint32_t)n_groups * kTileBytes);
                tma_load_3d(sm.a[s], &tm_a, &sm.full[s], kt * 64, I0, bh);
                for (int g = 0; g < n_groups; ++g)
                    tma_load_3d(sm.b[s] + g * kTileBytes, &tm_s, &sm.full[s], n0 + 64 * g, kt * 64, bh);
            }
        }
        if (!ok) {  // let in-flight loads land before the CTA exits
            for (int s = 0; s < kRedStages; ++s) {
                int jl = -1;
                for (int j = s; j < kc; j += kRedStages) jl = j;
                if (jl >= 0) mbar_wait_quiet(&sm.full[s], (jl / kRedStages) & 1);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        const uint64_t ad0 = sdesc_sw128(smem_u32(sm.a[0]), 16, 1024);
        const uint64_t bd0 = sdesc_sw128(smem_u32(sm.b[0]), kTileBytes, 1024);
        int kc = 0, lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++lt) {
            int bh, I0, n0;
            tile_coords(t, bh, I0, n0);
            const uint32_t id = idesc(1, 1, 1, 0, 1, 128, (uint32_t)min(256, kStateCols - n0));  // A K-, B MN-major
            const int buf = lt & 1;
            const uint32_t acc = tmem + 256 * buf;
            if (lt >= 2 && !(ok = mbar_wait(&sm.acc_empty[buf], ((lt >> 1) - 1) & 1, status, abort_flag))) break;
            tc_fence_after();
            for (int kt = 0; kt < nk; ++kt, ++kc) {
                const int s = kc % kRedStages, u = kc / kRedStages;
                if (!(ok = mbar_wait(&sm.full[s], u & 1, status, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(acc, dadd16(ad0, s * kRedA + 32 * k), dadd16(bd0, s * kRedB + 2048 * k), id,
                             (kt > 0 || k > 0) ? 1u : 0u);
                mma_commit(&sm.empty[s]);
            }
            if (!ok) break;
            mma_commit(&sm.acc_full[buf]);
        }
        mma_commit(&sm.drain);
        mbar_wait_quiet(&sm.drain, 0);  // MMAs retired before TMEM is freed
    } else if (warp >= 2) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        int lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++lt) {
            int bh, I0, n0;
            tile_coords(t, bh, I0, n0);
            const int n_valid = min(256, kStateCols - n0);
            const int buf = lt & 1;
            // global-state columns of this tile (subtract mode), staged per warp so that only
            // warp-local synchronisation is needed
            float *ht = sm.ht[q];
            if (subtract) {
                __syncwarp();
                for (int c = lane; c < n_valid; c += 32) ht[c] = __ldg(htot + (size_t)bh * kStateCols + n0 + c);
                __syncwarp();
            }
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_full[buf], (lt >> 1) & 1, status, abort_flag))))
                break;
            tc_fence_after();
            const int I = I0 + q * 32 + lane;
            float *dst = hq + ((size_t)bh * n_qb + I) * kStateCols + n0;
            const uint32_t acc = tmem + 256 * buf + ((uint32_t)(q * 32) << 16);
            for (int c0 = 0; c0 < n_valid; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(acc + c0, r);
                tmem_wait_ld();
                if (I < n_qb) {
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        float x = __uint_as_float(r[i]);
                        if (subtract) x = ht[c0 + i] - x;
                        v[i] = (n0 + c0 + i < kD * kD) ? to_tf32(x) : x;
                    }
                    float4 *o = reinterpret_cast<float4 *>(dst + c0);
#pragma unroll
                    for (int i = 0; i < 8; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
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

cudaError_t launch_states(const void *k, const void *v, const Geometry &g, int phi, uint16_t *states, float *partials,
                          uint16_t *v16, int *status, cudaStream_t s)
{
    CUtensorMap tk, tv;
    const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)g.N, (uint64_t)g.BH};
    const uint64_t strides[2] = {(uint64_t)kD * 2, (uint64_t)g.N * kD * 2};
    const uint32_t box[3] = {64, 64, 1};
    if (!encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dims, strides, box)) return cudaErrorInvalidValue;
    if (!encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dims, strides, box)) return cudaErrorInvalidValue;
    // at most two CTAs per SM: each holds 256 of the SM's 512 TMEM columns
    const size_t smem = sizeof(StatesSmem) + 1024 > 100 * 1024 ? sizeof(StatesSmem) + 1024 : 100 * 1024;
    cudaError_t e = cudaFuncSetAttribute(states_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(g.n_chunks, g.BH);
    states_kernel<<<grid, kStatesThreads, smem, s>>>(tk, tv, g.N, g.n_kb, g.n_chunks, phi, states, partials, v16,
                                                     status);
    return cudaGetLastError();
}

cudaError_t launch_htot(const float *partials, const Geometry &g, float *htot, cudaStream_t s)
{
    dim3 grid((kStateCols + 255) / 256, g.BH);
    htot_kernel<<<grid, 256, 0, s>>>(partials, g.n_chunks, htot);
    return cudaGetLastError();
}

cudaError_t launch_state_reduce(const uint16_t *amask, const uint16_t *states, const float *htot, const Geometry &g,
                                float *hq, int *status, cudaStream_t s)
{
    CUtensorMap ta, ts;
    {
        const uint64_t dims[3] = {(uint64_t)g.n_kb_pad, (uint64_t)g.n_qb, (uint64_t)g.BH};
        const uint64_t strides[2] = {(uint64_t)g.n_kb_pad * 2, (uint64_t)g.n_qb * g.n_kb_pad * 2};
        const uint32_t box[3] = {64, 128, 1};
        if (!encode_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, amask, dims, strides, box))
            return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[3] = {(uint64_t)kStateCols, (uint64_t)g.n_kb, (uint64_t)g.BH};
        const uint64_t strides[2] = {(uint64_t)kStateCols * 2, (uint64_t)g.n_kb * kStateCols * 2};
        const uint32_t box[3] = {64, 64, 1};
        if (!encode_tmap(&ts, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, states, dims, strides, box))
            return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(ReduceSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_tiles = g.BH * ((g.n_qb + 127) / 128) * ((kStateCols + 255) / 256);
    reduce_kernel<<<n_tiles < sms ? n_tiles : sms, kRedThreads, smem, s>>>(ta, ts, g.n_qb, g.n_kb, n_tiles,
                                                                         g.subtract ? 1 : 0, htot, hq, status);
    return cudaGetLastError();
}

}  // namespace sla
