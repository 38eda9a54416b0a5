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
//                 (M = 128 query blocks, N = 192 state columns, K = key
//                 blocks) with a 0/1 mask A, expanded from bits into tensor
//                 memory.  When at most half the key blocks
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

constexpr uint32_t kTileBytes = 64 * 128;  // one [64 rows x 128 B] TMA box

// ---------------------------------------------------------------------------
// per-key-block states: persistent, one CTA per SM over (bh, chunk of 32 key
// blocks) items.  Warp 0 = TMA producer (4 stages of K and V), warp 1 = MMA
// issuer, warps 2..5 = epilogue (TMEM lane quarter = warp index % 4), warps
// 6..13 = converters (phi(K) and V to fp16 in place, z_J by warp shuffles).
// TMEM: two per-block accumulators and two chunk-sum accumulators, so the
// epilogue of block J overlaps the MMAs of block J+1 and the chunk sum of one
// item is read while the next item accumulates.  The epilogue writes h_J^T
// through a swizzled shared stage and TMA tensor stores (one per warp slice).
// ---------------------------------------------------------------------------
constexpr int kStatesThreads = 448;
constexpr int kStStages = 4;

struct StatesSmem {
    alignas(1024) uint8_t kv[kStStages][4][kTileBytes];  // per stage: K channels 0-63, 64-127; V dims 0-63, 64-127
    alignas(1024) uint8_t out[2][2][2 * kTileBytes];     // [buffer][channel half]: 128 dims x 128 B, SW128
    uint64_t full[kStStages], conv[kStStages], empty[kStStages];
    uint64_t acc_full[2], acc_empty[2], sum_full[2], sum_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ float phi_f(float x, int phi)
{
    if (phi == 1) return fmaxf(x, 0.0f);
    const float e = ex2_approx(fminf(x, 0.0f) * 1.4426950408889634f);  // unconditional: a select, no branch
    return x > 0.0f ? x + 1.0f : e;  // rounded to fp16 next
}

__global__ void __launch_bounds__(kStatesThreads, 1) states_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                                   const __grid_constant__ CUtensorMap tm_v,
                                                                   const __grid_constant__ CUtensorMap tm_out, int N,
                                                                   int n_kb, int n_chunks, int n_items, int phi,
                                                                   uint16_t *__restrict__ states,
                                                                   float *__restrict__ partials,
                                                                   uint16_t *__restrict__ v16, int *status)
{
    extern __shared__ uint8_t smem_raw[];
    StatesSmem &sm = *reinterpret_cast<StatesSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int *abort_flag = &sm.abort_flag;
    if (tid == 0) sm.abort_flag = global_failed(status) ? 1 : 0;
    __syncthreads();
    if (sm.abort_flag) return;  // another CTA already failed: CTA-uniform early exit

    if (tid == 0) {
        for (int s = 0; s < kStStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.conv[s], 256);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 128);
            mbar_init(&sm.sum_full[b], 1);
            mbar_init(&sm.sum_empty[b], 128);
        }
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_out);
    }
    __syncwarp();
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;  // [0,256): block accumulators, [256,512): chunk sums

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int j = 0;  // blocks issued by this CTA
            bool ok = true;
            for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
                const int bh = it / n_chunks, Jbeg = (it % n_chunks) * kStateChunk;
                const int nJ = min(kStateChunk, n_kb - Jbeg);
                for (int jj = 0; jj < nJ; ++jj, ++j) {
                    const int s = j % kStStages, u = j / kStStages, row = (Jbeg + jj) * 64;
                    if (u > 0 && !(ok = mbar_wait(&sm.empty[s], (u - 1) & 1, status, abort_flag))) break;
                    mbar_expect_tx(&sm.full[s], 4 * kTileBytes);
                    tma_load_4d(sm.kv[s][0], &tm_k, &sm.full[s], 0, row, 0, bh);  // both halves of K
                    tma_load_4d(sm.kv[s][2], &tm_v, &sm.full[s], 0, row, 0, bh);  // both halves of V
                }
            }
            if (!ok) {  // loads in flight land before the CTA exits
                for (int s = 0; s < kStStages; ++s) {
                    int jl = -1;
                    for (int x = s; x < j; x += kStStages) jl = x;
                    if (jl >= 0) mbar_wait_quiet(&sm.full[s], (jl / kStStages) & 1, status);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdesc = idesc(1, 0, 0, 1, 1, 128, 128);  // f32 <- f16 (MN) x f16 (MN)
            const uint64_t vd0 = sdesc_sw128(smem_u32(sm.kv[0][2]), kTileBytes, 1024);  // A = V^T (dims x tokens)
            const uint64_t kd0 = sdesc_sw128(smem_u32(sm.kv[0][0]), kTileBytes, 1024);  // B = phi(K) (ch x tokens)
            constexpr uint32_t kStage16 = 4 * kTileBytes >> 4;
            int j = 0, li = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++li) {
                const int Jbeg = (it % n_chunks) * kStateChunk, nJ = min(kStateChunk, n_kb - Jbeg);
                const int cb = li & 1;
                const uint32_t d_sum = tmem + 256 + 128 * cb;
                if (li >= 2 && !(ok = mbar_wait(&sm.sum_empty[cb], ((li >> 1) - 1) & 1, status, abort_flag))) break;
                for (int jj = 0; jj < nJ; ++jj, ++j) {
                    const int s = j % kStStages, b = j & 1;
                    const uint32_t d_blk = tmem + 128 * b;
                    if (j >= 2 && !(ok = mbar_wait(&sm.acc_empty[b], ((j >> 1) - 1) & 1, status, abort_flag))) break;
                    if (!(ok = mbar_wait(&sm.conv[s], (j / kStStages) & 1, status, abort_flag))) break;
                    tc_fence_after();
                    const uint64_t vd = vd0 + (uint64_t)(s * kStage16), kd = kd0 + (uint64_t)(s * kStage16);
#pragma unroll
                    for (int k = 0; k < 4; ++k) mma_bf16(d_blk, vd + 128 * k, kd + 128 * k, kIdesc, k > 0 ? 1u : 0u);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(d_sum, vd + 128 * k, kd + 128 * k, kIdesc, (jj > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&sm.empty[s]);
                    mma_commit(&sm.acc_full[b]);
                    if (jj == nJ - 1) mma_commit(&sm.sum_full[cb]);
                }
            }
            mma_commit(&sm.drain);
            mbar_wait_quiet(&sm.drain, 0, status);  // MMAs retired before TMEM is freed
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3, d = 32 * q + lane;  // TMEM lane = dim row of h_J^T
        int j = 0, li = 0;
        bool ok = true;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++li) {
            const int bh = it / n_chunks, chunk = it % n_chunks, Jbeg = chunk * kStateChunk;
            const int nJ = min(kStateChunk, n_kb - Jbeg), cb = li & 1;
            for (int jj = 0; jj < nJ; ++jj, ++j) {
                const int b = j & 1;
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_full[b], (j >> 1) & 1, status, abort_flag))))
                    break;
                tc_fence_after();
                if (lane == 0) bulk_wait_read<1>();  // the store issued from this buffer two blocks ago has read it
                __syncwarp();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {  // channel half: two 32-column loads, one wait
                    uint32_t r[64];
                    const uint32_t ta = tmem + 128 * b + ((uint32_t)(32 * q) << 16) + 64 * hh;
                    tmem_ld32(ta, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
                    tmem_ld32(ta + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
                    tmem_wait_ld();
                    uint8_t *row = sm.out[b][hh] + d * 128;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        *reinterpret_cast<uint4 *>(row + ((u ^ (d & 7)) << 4)) =
                            make_uint4(pack_bf16x2(__uint_as_float(r[8 * u]), __uint_as_float(r[8 * u + 1])),
                                       pack_bf16x2(__uint_as_float(r[8 * u + 2]), __uint_as_float(r[8 * u + 3])),
                                       pack_bf16x2(__uint_as_float(r[8 * u + 4]), __uint_as_float(r[8 * u + 5])),
                                       pack_bf16x2(__uint_as_float(r[8 * u + 6]), __uint_as_float(r[8 * u + 7])));
                }
                tc_fence_before();
                mbar_arrive(&sm.acc_empty[b]);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int blk = bh * n_kb + Jbeg + jj;
                    tma_store_3d(&tm_out, sm.out[b][0] + 32 * q * 128, 0, 32 * q, blk);
                    tma_store_3d(&tm_out, sm.out[b][1] + 32 * q * 128, 64, 32 * q, blk);
                    bulk_commit();
                }
            }
            if (!ok) break;
            // chunk sum of the fp32 states
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.sum_full[cb], (li >> 1) & 1, status, abort_flag))))
                break;
            tc_fence_after();
            float *dst = partials + ((size_t)bh * n_chunks + chunk) * kStateCols + (size_t)d * kD;
#pragma unroll 1
            for (int c0 = 0; c0 < kD; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(tmem + 256 + 128 * cb + ((uint32_t)(32 * q) << 16) + c0, r);
                tmem_wait_ld();
                float4 *o = reinterpret_cast<float4 *>(dst + c0);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    o[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                       __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
            }
            tc_fence_before();
            mbar_arrive(&sm.sum_empty[cb]);
        }
        if (lane == 0) bulk_wait<0>();  // stores complete before shared memory is released
    } else {
        // ------------------------------------------------------------ converters
        // thread -> (channel half, 16-byte unit u, row group rg): rows rg + 16i of unit u,
        // whose swizzled position is u ^ (rg & 7); lanes rg = 0..15 reduce z by shuffles
        const int ct = tid - 192, cw = ct >> 5, rg = lane & 15;
        const int half = cw >> 2, u = (cw & 3) * 2 + (lane >> 4);
        const int ch0 = half * 64 + u * 8;  // first of this thread's 8 channels
        const uint32_t off0 = rg * 128 + ((u ^ (rg & 7)) << 4);
        int j = 0;
        bool ok = true;
        for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
            const int bh = it / n_chunks, chunk = it % n_chunks, Jbeg = chunk * kStateChunk;
            const int nJ = min(kStateChunk, n_kb - Jbeg);
            float zc[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // chunk sums of z (lanes rg == 0)
            for (int jj = 0; jj < nJ; ++jj, ++j) {
                const int s = j % kStStages, J = Jbeg + jj;
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.full[s], (j / kStStages) & 1, status, abort_flag))))
                    break;
                const int valid = min(64, N - J * 64);  // tokens past N contribute nothing
                float z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                uint4 wk[4], wv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    wk[i] = *reinterpret_cast<const uint4 *>(sm.kv[s][half] + off0 + i * 2048);
                    wv[i] = *reinterpret_cast<const uint4 *>(sm.kv[s][2 + half] + off0 + i * 2048);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = rg + 16 * i;
                    const uint32_t kk[4] = {wk[i].x, wk[i].y, wk[i].z, wk[i].w};
                    const uint32_t vv[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
                    uint32_t ok4[4], ov4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float a = phi_f(__uint_as_float(kk[e] << 16), phi);
                        const float c = phi_f(__uint_as_float(kk[e] & 0xFFFF0000u), phi);
                        ok4[e] = r < valid ? pack_f16x2_sat(a, c) : 0u;
                        ov4[e] = r < valid ? pack_f16x2_sat(__uint_as_float(vv[e] << 16),
                                                            __uint_as_float(vv[e] & 0xFFFF0000u))
                                           : 0u;
                        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&ok4[e]));
                        z[2 * e] += f.x;
                        z[2 * e + 1] += f.y;
                    }
                    *reinterpret_cast<uint4 *>(sm.kv[s][half] + off0 + i * 2048) =
                        make_uint4(ok4[0], ok4[1], ok4[2], ok4[3]);
                    *reinterpret_cast<uint4 *>(sm.kv[s][2 + half] + off0 + i * 2048) =
                        make_uint4(ov4[0], ov4[1], ov4[2], ov4[3]);
                    if (v16 != nullptr && r < valid)  // fp16 copy of V for the attention kernel's fp16 P.V
                        *reinterpret_cast<uint4 *>(v16 + ((size_t)bh * N + J * 64 + r) * kD + ch0) =
                            make_uint4(ov4[0], ov4[1], ov4[2], ov4[3]);
                }
                fence_async_smem();
                mbar_arrive(&sm.conv[s]);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
#pragma unroll
                    for (int o = 1; o < 16; o <<= 1) z[e] += __shfl_xor_sync(0xffffffffu, z[e], o);
                }
                if (rg == 0) {
                    *reinterpret_cast<uint4 *>(states + ((size_t)bh * n_kb + J) * kStateCols + kD * kD + ch0) =
                        make_uint4(pack_bf16x2(z[0], z[1]), pack_bf16x2(z[2], z[3]), pack_bf16x2(z[4], z[5]),
                                   pack_bf16x2(z[6], z[7]));
#pragma unroll
                    for (int e = 0; e < 8; ++e) zc[e] += z[e];
                }
            }
            if (!ok) break;
            if (rg == 0) {
                float4 *o = reinterpret_cast<float4 *>(partials + ((size_t)bh * n_chunks + chunk) * kStateCols +
                                                       kD * kD + ch0);
                o[0] = make_float4(zc[0], zc[1], zc[2], zc[3]);
                o[1] = make_float4(zc[4], zc[5], zc[6], zc[7]);
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
// per-query-block state: persistent GEMM over tiles (bh, 192 state columns,
// 128 query blocks), m fastest so the query-block tiles of one column tile run
// together and share the state columns through L2.  The 0/1 mask never goes
// through shared memory: top-k writes it as bits, and four builder warps expand
// each row's 64 bits of a k-step into bf16 pairs stored straight into tensor
// memory, where the MMA takes its A operand.  Only the states (B, MN-major)
// stream in by TMA, 24 KB per k-step.
//   warp 0      TMA producer (B ring, kRedBStages)
//   warp 1      MMA issuer
//   warps 2..5  epilogue (TMEM lane quarter = warp index % 4): 32 x 32 fp32
//               chunks staged swizzled in shared memory and written by TMA stores
//   warps 6..9  A builders (same lane quarters)
// TMEM: two accumulators [0, 384) so the epilogue of one tile overlaps the
// next tile's MMAs, and the A ring [384, 512): kRedAStages x 32 columns (one
// k-step of 64 key blocks as 16-bit pairs).  16512 state columns = 86 x 192.
// ---------------------------------------------------------------------------
constexpr int kRedBStages = 6;
constexpr int kRedAStages = 4;
constexpr int kRedThreads = 320;
constexpr int kRedN = 192;
constexpr uint32_t kRedB = 3 * kTileBytes;  // 64 key blocks x 192 columns (bf16), three 64-column boxes
constexpr uint32_t kRedACol = 2 * kRedN;    // first TMEM column of the A ring
constexpr int kRedEpiBufs = 3;              // 4 KB output staging buffers per epilogue warp
static_assert(kStateCols % kRedN == 0, "state columns split into whole tiles");
static_assert(kRedACol + 32 * kRedAStages <= 512, "TMEM budget");

struct ReduceSmem {
    alignas(1024) uint8_t b[kRedBStages][kRedB];
    alignas(1024) uint8_t out[4][kRedEpiBufs][32 * 128];  // [epilogue warp][buffer]: 32 rows x 32 fp32, SW128
    float ht[4][kRedN];  // global-state columns of the tile in the epilogue, one copy per epilogue warp
    uint64_t full[kRedBStages], empty[kRedBStages];
    uint64_t a_full[kRedAStages], a_empty[kRedAStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ uint64_t dadd16(uint64_t desc, uint32_t bytes) { return desc + (uint64_t)(bytes >> 4); }

// bf16 MMA with A in tensor memory (rows = lanes, two K elements per 32-bit column, the lower K
// in the low half)
__device__ __forceinline__ void mma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc_,
                                                uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc_), "r"(accumulate)
        : "memory");
}

// the mask words of k-steps kt .. kt+3 of one row (zeros past the row's end or for a padding row)
__device__ __forceinline__ void load_mask4(const uint32_t *row, int kt, int nk, uint32_t (&w)[8])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint2 v = make_uint2(0u, 0u);
        if (row && kt + i < nk) v = __ldg(reinterpret_cast<const uint2 *>(row) + kt + i);
        w[2 * i] = v.x;
        w[2 * i + 1] = v.y;
    }
}

__global__ void __launch_bounds__(kRedThreads, 1) reduce_kernel(const uint32_t *__restrict__ amask, int n_aw,
                                                                const __grid_constant__ CUtensorMap tm_s,
                                                                const __grid_constant__ CUtensorMap tm_hq, int n_qb,
                                                                int n_kb, int n_tiles, int subtract,
                                                                const float *__restrict__ htot, int *status)
{
    extern __shared__ uint8_t smem_raw[];
    ReduceSmem &sm = *reinterpret_cast<ReduceSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_mt = (n_qb + 127) / 128, n_nt = kStateCols / kRedN;
    const int nk = (n_kb + 63) / 64;
    volatile int *abort_flag = &sm.abort_flag;
    if (tid == 0) sm.abort_flag = global_failed(status) ? 1 : 0;
    __syncthreads();
    if (sm.abort_flag) return;  // another CTA already failed: CTA-uniform early exit

    if (tid == 0) {
        for (int s = 0; s < kRedBStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int s = 0; s < kRedAStages; ++s) {
            mbar_init(&sm.a_full[s], 128);
            mbar_init(&sm.a_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 128);
        }
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_s);
        tma_prefetch_desc(&tm_hq);
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
        n0 = (rest % n_nt) * kRedN;
        I0 = m * 128;
    };

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ producer (states)
        int kc = 0;  // k-steps issued over all tiles of this CTA
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
            int bh, I0, n0;
            tile_coords(t, bh, I0, n0);
            for (int kt = 0; kt < nk; ++kt, ++kc) {
                const int s = kc % kRedBStages, u = kc / kRedBStages;
                if (u > 0 && !(ok = mbar_wait(&sm.empty[s], (u - 1) & 1, status, abort_flag))) break;
                mbar_expect_tx(&sm.full[s], kRedB);
                tma_load_4d(sm.b[s], &tm_s, &sm.full[s], n0, kt * 64, 0, bh);  // the three 64-column groups
            }
        }
        if (!ok) {  // let in-flight loads land before the CTA exits
            for (int s = 0; s < kRedBStages; ++s) {
                int jl = -1;
                for (int j = s; j < kc; j += kRedBStages) jl = j;
                if (jl >= 0) mbar_wait_quiet(&sm.full[s], (jl / kRedBStages) & 1, status);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        const uint64_t bd0 = sdesc_sw128(smem_u32(sm.b[0]), kTileBytes, 1024);
        const uint32_t id = idesc(1, 1, 1, 0, 1, 128, kRedN);  // A from TMEM, B MN-major
        int kc = 0, lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++lt) {
            const int buf = lt & 1;
            const uint32_t acc = tmem + kRedN * buf;
            if (lt >= 2 && !(ok = mbar_wait(&sm.acc_empty[buf], ((lt >> 1) - 1) & 1, status, abort_flag))) break;
            tc_fence_after();
            for (int kt = 0; kt < nk; ++kt, ++kc) {
                const int sb = kc % kRedBStages, sa = kc % kRedAStages;
                const uint32_t pa = (kc / kRedAStages) & 1, pb = (kc / kRedBStages) & 1;
                const bool ra = mbar_test(&sm.a_full[sa], pa);  // both tests in flight together
                const bool rb = mbar_test(&sm.full[sb], pb);
                if (!ra && !(ok = mbar_wait(&sm.a_full[sa], pa, status, abort_flag))) break;
                if (!rb && !(ok = mbar_wait(&sm.full[sb], pb, status, abort_flag))) break;
                tc_fence_after();
                const uint32_t a_t = tmem + kRedACol + 32 * sa;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16_tmem_a(acc, a_t + 8 * k, dadd16(bd0, sb * kRedB + 2048 * k), id,
                                    (kt > 0 || k > 0) ? 1u : 0u);
                mma_commit(&sm.empty[sb]);
                mma_commit(&sm.a_empty[sa]);
            }
            if (!ok) break;
            mma_commit(&sm.acc_full[buf]);
        }
        mma_commit(&sm.drain);
        mbar_wait_quiet(&sm.drain, 0, status);  // MMAs retired before TMEM is freed
    } else if (warp >= 6) {
        // ------------------------------------------------------------ A builders
        // Thread = one query block (TMEM lane); column c of a k-step holds the mask of key
        // blocks 64 kt + 2c (low half) and 64 kt + 2c + 1 (high half): bf16 1.0 or 0.
        const int q = warp & 3;
        const uint32_t a_lane = (uint32_t)(q * 32) << 16;
        auto row_of = [&](int t) -> const uint32_t * {
            if (t >= n_tiles) return nullptr;
            int bh, I0, n0;
            tile_coords(t, bh, I0, n0);
            const int I = I0 + q * 32 + lane;
            return I < n_qb ? amask + ((size_t)bh * n_qb + I) * n_aw : nullptr;
        };
        int kc = 0;
        bool ok = true;
        uint32_t w[8];
        load_mask4(row_of(blockIdx.x), 0, nk, w);
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
            const uint32_t *row = row_of(t), *next_row = row_of(t + gridDim.x);
            for (int kt0 = 0; ok && kt0 < nk; kt0 += 4) {
                uint32_t nx[8];  // one group ahead, into the next tile at the end of this one
                if (kt0 + 4 < nk)
                    load_mask4(row, kt0 + 4, nk, nx);
                else
                    load_mask4(next_row, 0, nk, nx);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (kt0 + j < nk) {  // warp-uniform
                        const int sa = kc % kRedAStages, u = kc / kRedAStages;
                        if (u > 0 && !(ok = mbar_wait_warp(&sm.a_empty[sa], (u - 1) & 1, status, abort_flag)))
                            break;
                        tc_fence_after();
                        uint32_t r[32];
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const uint32_t b = (w[2 * j + (c >> 4)] >> (2 * (c & 15))) & 3u;
                            r[c] = (b & 1u) * 0x3F80u + (b >> 1) * 0x3F800000u;
                        }
                        tmem_st32(tmem + a_lane + kRedACol + 32 * sa, r);
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&sm.a_full[sa]);
                        ++kc;
                    }
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) w[i] = nx[i];
            }
        }
    } else if (warp >= 2) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        int lt = 0, ec = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++lt) {
            int bh, I0, n0;
            tile_coords(t, bh, I0, n0);
            const int buf = lt & 1;
            // global-state columns of this tile (subtract mode), staged per warp so that only
            // warp-local synchronisation is needed
            float *ht = sm.ht[q];
            if (subtract) {
                __syncwarp();
                for (int c = lane; c < kRedN; c += 32) ht[c] = __ldg(htot + (size_t)bh * kStateCols + n0 + c);
                __syncwarp();
            }
            if (!(ok = mbar_wait_warp(&sm.acc_full[buf], (lt >> 1) & 1, status, abort_flag))) break;
            tc_fence_after();
            const uint32_t acc = tmem + kRedN * buf + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
            for (int c0 = 0; c0 < kRedN; c0 += 32, ++ec) {
                uint32_t r[32];
                tmem_ld32(acc + c0, r);
                tmem_wait_ld();
                if (c0 + 32 == kRedN) {  // the accumulator is read: the next tile may start on it
                    tc_fence_before();
                    mbar_arrive(&sm.acc_empty[buf]);
                }
                uint8_t *stage = sm.out[q][ec % kRedEpiBufs];
                if (lane == 0) bulk_wait_read<kRedEpiBufs - 1>();  // the store that used this buffer has read it
                __syncwarp();
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    float v[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c = c0 + 4 * u + i;
                        float x = __uint_as_float(r[4 * u + i]);
                        if (subtract) x = ht[c] - x;
                        v[i] = (n0 + c < kD * kD) ? to_tf32(x) : x;
                    }
                    *reinterpret_cast<float4 *>(stage + lane * 128 + ((u ^ (lane & 7)) << 4)) =
                        make_float4(v[0], v[1], v[2], v[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {  // rows past n_qb fall outside the tensor map and are not written
                    tma_store_3d(&tm_hq, stage, n0 + c0, I0 + 32 * q, bh);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait<0>();  // stores complete before the CTA exits
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
    CUtensorMap tk, tv, to;
    // K and V [BH, N, 128] viewed as [64 elements, N rows (256 B apart), 2 halves (128 B apart), BH]:
    // one box per key block lands as its two [64 rows x 128 B] half-tiles, one after the other
    const uint64_t dims[4] = {64, (uint64_t)g.N, 2, (uint64_t)g.BH};
    const uint64_t strides[3] = {(uint64_t)kD * 2, 128, (uint64_t)g.N * kD * 2};
    const uint32_t box[4] = {64, 64, 2, 1};
    if (!encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, k, dims, strides, box)) return cudaErrorInvalidValue;
    if (!encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, v, dims, strides, box)) return cudaErrorInvalidValue;
    {
        // h_J^T of every key block: [BH * n_kb][128 dims][128 channels] inside rows of kStateCols
        const uint64_t od[3] = {(uint64_t)kD, (uint64_t)kD, (uint64_t)g.BH * g.n_kb};
        const uint64_t os[2] = {(uint64_t)kD * 2, (uint64_t)kStateCols * 2};
        const uint32_t ob[3] = {64, 32, 1};
        if (!encode_tmap(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, states, od, os, ob)) return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(StatesSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(states_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_items = g.BH * g.n_chunks;
    states_kernel<<<n_items < sms ? n_items : sms, kStatesThreads, smem, s>>>(tk, tv, to, g.N, g.n_kb, g.n_chunks,
                                                                             n_items, phi, states, partials, v16,
                                                                             status);
    return cudaGetLastError();
}

cudaError_t launch_htot(const float *partials, const Geometry &g, float *htot, cudaStream_t s)
{
    dim3 grid((kStateCols + 255) / 256, g.BH);
    htot_kernel<<<grid, 256, 0, s>>>(partials, g.n_chunks, htot);
    return cudaGetLastError();
}

cudaError_t launch_state_reduce(const uint32_t *amask, const uint16_t *states, const float *htot, const Geometry &g,
                                float *hq, int *status, cudaStream_t s)
{
    if (g.n_aw != 2 * ((g.n_kb + 63) / 64)) return cudaErrorInvalidValue;
    CUtensorMap ts, th;
    {
        const uint64_t dims[3] = {(uint64_t)kStateCols, (uint64_t)g.n_qb, (uint64_t)g.BH};
        const uint64_t strides[2] = {(uint64_t)kStateCols * 4, (uint64_t)g.n_qb * kStateCols * 4};
        const uint32_t box[3] = {32, 32, 1};
        if (!encode_tmap(&th, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, hq, dims, strides, box))
            return cudaErrorInvalidValue;
    }
    {
        // states [BH][n_kb][kStateCols] bf16 viewed as [columns, key blocks, 3 column groups (128 B
        // apart), BH]: a box of {64, 64, 3, 1} at column n0 holds columns n0 + 64 g + (0..63) for g < 3,
        // landing as the three [64 key blocks x 128 B] tiles of a k-step one after the other (the
        // group dimension overlaps the column dimension; the box never leaves the row: n0 + 191 <
        // kStateCols)
        const uint64_t dims[4] = {(uint64_t)kStateCols, (uint64_t)g.n_kb, 3, (uint64_t)g.BH};
        const uint64_t strides[3] = {(uint64_t)kStateCols * 2, 128, (uint64_t)g.n_kb * kStateCols * 2};
        const uint32_t box[4] = {64, 64, 3, 1};
        if (!encode_tmap(&ts, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, states, dims, strides, box))
            return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(ReduceSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_tiles = g.BH * ((g.n_qb + 127) / 128) * (kStateCols / kRedN);
    reduce_kernel<<<n_tiles < sms ? n_tiles : sms, kRedThreads, smem, s>>>(amask, g.n_aw, ts, th, g.n_qb, g.n_kb,
                                                                         n_tiles, g.subtract ? 1 : 0, htot, status);
    return cudaGetLastError();
}

cudaError_t set_wait_budget_linear(long long cycles) { return set_tu_wait_budget(cycles); }

}  // namespace sla
