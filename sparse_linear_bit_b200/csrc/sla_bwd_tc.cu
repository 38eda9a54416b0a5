// sla_bwd_tc.cu -- the softmax branch of the SageSLA backward on tcgen05
// tensor cores (SLA fine-tuning: the jiqiren.org.cn TurboDiffusion article,
// 方法论; the "TurboDiffusion" summary page, 主要能力: SLA white-box training).
//
// For row i of query block I and the tokens j of the key blocks I selected,
// with s = q.k / sqrt(d), p = softmax_j(s), dP = do.v, D_i = sum_j p_ij dP_ij:
//   dS_ij = p_ij (dP_ij - D_i) / sqrt(d);  dq_i = sum_j dS_ij k_j;
//   dv_j = sum_i p_ij do_i;                 dk_j = sum_i dS_ij q_i.
//
// bwdq_kernel, one CTA per (head, query block), two passes over the selected
// key blocks (K and V tiles stream through a TMA ring twice):
//   pass 1: S = Q K^T and dP = dO V^T into tensor memory; per row the online
//           max m, sum l and D (the softmax-weighted sum of dP), written out
//           for the key side;
//   pass 2: S and dP again; dS from them in fp32, rounded to bf16 into shared
//           memory, and dQ += dS K accumulated in tensor memory.  Since
//           sum_j dS_ij = 0, dq_i = sum_j dS_ij (k_j - mu) for any vector mu;
//           with mu = the head's mean key, the bf16 rounding of dS is not
//           multiplied by the keys' common component: the kernel sums, in
//           fp32, sigma_i = sum_j of the rounded dS_ij and writes
//           dq_i = (dS K)_i - sigma_i mu.
// bwdk_kernel, one CTA per (head, key block), over the query blocks that
//   selected it: S and dP as above, P and dS (from the row statistics of
//   pass 1) rounded to bf16 into shared memory, and dV^T += dO^T P,
//   dK^T += Q^T dS accumulated in tensor memory (M = 128 dims, N = 64 keys);
//   the results are added to dk, dv, which the linear branch's key side has
//   written before.
//
// Roles: warp 0 TMA producer, warp 1 MMA issuer and TMEM owner, then the row
// warps: in bwdq (192 threads) warps 2-5, one query row per thread; in bwdk (320
// threads) warps 2-9, two threads per query row, each with half of the tile's 64
// keys (in bwdk's epilogue, one dim or channel per pair, half of the keys each).
// All products take bf16 operands with fp32 accumulation.  Every wait is bounded
// (see sla_ptx.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sla_internal.h"
#include "sla_ptx.cuh"

namespace sla {
namespace {

constexpr int kBwThreads = 192;
constexpr int kBkThreads = 320;
constexpr uint32_t kBox = 64 * 128;    // [64 rows x 128 B]
constexpr uint32_t kTile = 128 * 128;  // [128 rows x 128 B]
constexpr int kBqStages = 4;
constexpr int kBkStages = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRsd = 0.08838834764831845f;  // 1 / sqrt(128)

SLA_DEV uint64_t dadd(uint64_t desc, uint32_t bytes) { return desc + (uint64_t)(bytes >> 4); }

SLA_DEV float ex2f(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

SLA_DEV void named_bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// 64 fp32 columns of this thread's TMEM lane
SLA_DEV void tmem_ld64(uint32_t taddr, uint32_t (&r)[64])
{
    tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}

// row r (64 bf16 = 128 B, packed in 32 words) of a [128 rows x 128 B] tile with the 128-byte swizzle
SLA_DEV void store_row_sw128(uint8_t *tile, int r, const uint32_t (&w)[32])
{
#pragma unroll
    for (int u = 0; u < 8; ++u)
        *reinterpret_cast<uint4 *>(tile + sw128_off(r, u)) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
}

// S and dP of one (query block, key block) tile: M = 128 query rows, N = 64 keys, K = 128 in
// 8 steps of 16 bf16.  A tiles (Q, dO) are [128 rows x 128 B] boxes, B tiles (K, V) [64 rows x 128 B]
// boxes, both K-major with the 128-byte swizzle, channels 0-63 then 64-127.
SLA_DEV void issue_s_dp(uint32_t t_s, uint32_t t_dp, uint64_t qd, uint64_t dod, uint64_t kd, uint64_t vd)
{
    constexpr uint32_t id = idesc(1, 1, 1, 0, 0, 128, 64);  // f32 <- bf16 x bf16
    // the two accumulation chains alternate, so that one chain's MMA overlaps the other's
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        mma_bf16(t_s, dadd(qd, (k >> 2) * kTile + (k & 3) * 32), dadd(kd, (k >> 2) * kBox + (k & 3) * 32), id,
                 k > 0 ? 1u : 0u);
        mma_bf16(t_dp, dadd(dod, (k >> 2) * kTile + (k & 3) * 32), dadd(vd, (k >> 2) * kBox + (k & 3) * 32), id,
                 k > 0 ? 1u : 0u);
    }
}

// ---------------------------------------------------------------------------
// query side
// ---------------------------------------------------------------------------
struct BqSmem {
    alignas(1024) uint8_t q[2 * kTile];              // Q_I: channels 0-63 | 64-127
    alignas(1024) uint8_t dO[2 * kTile];             // dO_I: dims 0-63 | 64-127
    alignas(1024) uint8_t kv[kBqStages][4][kBox];    // per stage: K_J ch 0-63 | 64-127, V_J dims 0-63 | 64-127
    alignas(1024) uint8_t ds[2][kTile];              // dS tiles: [128 rows x 64 keys] bf16
    float mu[128];
    uint64_t full[kBqStages], empty[kBqStages];
    uint64_t bar_qdo, bar_sd[2], bar_sdfree[2], bar_ds[2], bar_dsfree[2], bar_dq, drain;
    uint32_t tmem_base;
    int abort_flag;
};

__global__ void __launch_bounds__(kBwThreads, 1)
bwdq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
            const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
            const int32_t *__restrict__ idx, const float *__restrict__ kmean, int N, int blk_q, int n_qb, int k_sel,
            float *__restrict__ dq, float *__restrict__ st_m, float *__restrict__ st_l, float *__restrict__ st_D,
            int *status)
{
    extern __shared__ uint8_t smem_raw[];
    BqSmem &sm = *reinterpret_cast<BqSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int I = blockIdx.x, bh = blockIdx.y;
    const int32_t *sel = idx + ((size_t)bh * n_qb + I) * k_sel;
    const int nT = 2 * k_sel;  // tiles: pass 1 (T < k_sel), then pass 2
    volatile int *abort_flag = &sm.abort_flag;
    if (tid == 0) sm.abort_flag = global_failed(status) ? 1 : 0;
    __syncthreads();
    if (sm.abort_flag) return;  // another CTA already failed: CTA-uniform early exit

    if (tid == 0) {
        for (int s = 0; s < kBqStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.bar_qdo, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.bar_sd[b], 1);
            mbar_init(&sm.bar_sdfree[b], 128);
            mbar_init(&sm.bar_ds[b], 128);
            mbar_init(&sm.bar_dsfree[b], 1);
        }
        mbar_init(&sm.bar_dq, 1);
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;  // S / dP of buffer b at 128 b / 128 b + 64; dQ at 256
    const uint32_t t_dq = tmem + 256;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (elect_one()) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_do);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_expect_tx(&sm.bar_qdo, 4 * kTile);
            tma_load_4d(sm.q, &tm_q, &sm.bar_qdo, 0, I * blk_q, 0, bh);
            tma_load_4d(sm.dO, &tm_do, &sm.bar_qdo, 0, I * blk_q, 0, bh);
        }
        __syncwarp();
        int issued = 0;
        bool ok = true;
        for (int T = 0; ok && T < nT; ++T) {
            const int s = T % kBqStages, u = T / kBqStages;
            if (u > 0 && !(ok = mbar_wait_warp(&sm.empty[s], (u - 1) & 1, status, abort_flag))) break;
            const int J = __ldg(sel + (T < k_sel ? T : T - k_sel));
            if (elect_one()) {
                mbar_expect_tx(&sm.full[s], 4 * kBox);
                tma_load_4d(sm.kv[s][0], &tm_k, &sm.full[s], 0, J * 64, 0, bh);
                tma_load_4d(sm.kv[s][2], &tm_v, &sm.full[s], 0, J * 64, 0, bh);
            }
            __syncwarp();
            issued = T + 1;
        }
        // every load issued has landed before shared memory is released
        for (int s = 0; s < kBqStages; ++s) {
            int tl = -1;
            for (int T = s; T < issued; T += kBqStages) tl = T;
            if (tl >= 0) mbar_wait_quiet(&sm.full[s], (tl / kBqStages) & 1, status);
        }
        mbar_wait_quiet(&sm.bar_qdo, 0, status);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t id_dq = idesc(1, 1, 1, 0, 1, 128, 128);  // A = dS K-major, B = K MN-major
        const uint64_t qd = sdesc_sw128(smem_u32(sm.q), 16, 1024), dod = sdesc_sw128(smem_u32(sm.dO), 16, 1024);
        bool ok = k_sel == 0 || mbar_wait_warp(&sm.bar_qdo, 0, status, abort_flag);
        // both issue steps run once the poll below has seen their barriers' phases complete
        auto issue_sd = [&](int T) {
            const int s = T % kBqStages, b = T & 1;
            tc_fence_after();
            if (elect_one()) {
                issue_s_dp(tmem + 128 * b, tmem + 128 * b + 64, qd, dod, sdesc_sw128(smem_u32(sm.kv[s][0]), 16, 1024),
                           sdesc_sw128(smem_u32(sm.kv[s][2]), 16, 1024));
                mma_commit(&sm.bar_sd[b]);
                if (T < k_sel) mma_commit(&sm.empty[s]);  // pass 1: the stage is free after S and dP
            }
            __syncwarp();
        };
        auto issue_dq = [&](int t) {  // pass-2 tile t
            const int T = k_sel + t, s = T % kBqStages, b = t & 1;
            tc_fence_after();
            if (elect_one()) {
                const uint64_t dsd = sdesc_sw128(smem_u32(sm.ds[b]), 16, 1024);
                const uint64_t kmn = sdesc_sw128(smem_u32(sm.kv[s][0]), kBox, 1024);
#pragma unroll
                for (int k = 0; k < 4; ++k)  // K-step of 16 keys: 32 B of a dS row, 2 KB of K rows
                    mma_bf16(t_dq, dadd(dsd, 32 * k), dadd(kmn, 2048 * k), id_dq, (t > 0 || k > 0) ? 1u : 0u);
                mma_commit(&sm.bar_dsfree[b]);
                mma_commit(&sm.empty[s]);
                if (t == k_sel - 1) mma_commit(&sm.bar_dq);
            }
            __syncwarp();
        };
        // dQ of a pass-2 tile is issued as soon as its dS is in shared memory (it frees a K/V stage
        // and a dS buffer); S/dP of the next tile as soon as its stage has landed and its TMEM
        // buffer is free
        int n_sd = 0, n_dq = 0;
        long long t0c = clock64();
        const long long budget = wait_budget();
        while (ok && n_dq < k_sel) {
            const bool can_dq = n_dq < n_sd - k_sel && mbar_test(&sm.bar_ds[n_dq & 1], (n_dq >> 1) & 1);
            if (__any_sync(0xffffffffu, can_dq)) {
                issue_dq(n_dq++);
                t0c = clock64();
                continue;
            }
            const bool can_sd = n_sd < nT && mbar_test(&sm.full[n_sd % kBqStages], (n_sd / kBqStages) & 1) &&
                                (n_sd < 2 || mbar_test(&sm.bar_sdfree[n_sd & 1], ((n_sd >> 1) - 1) & 1));
            if (__any_sync(0xffffffffu, can_sd)) {
                issue_sd(n_sd++);
                t0c = clock64();
                continue;
            }
            if (clock64() - t0c > budget) {  // neither came: the same bounded-wait rule as mbar_wait
                if (elect_one()) record_error(status, kStatusTimeout);
                *abort_flag = 1;
                ok = false;
            } else if (global_failed(status) || *abort_flag) {
                *abort_flag = 1;
                ok = false;
            }
            ok = __all_sync(0xffffffffu, ok);
        }
        if (elect_one()) {
            mma_commit(&sm.drain);
            mbar_wait_quiet(&sm.drain, 0, status);  // this thread's MMAs retired before TMEM is released
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ rows
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int i = I * blk_q + r;
        const bool row_valid = r < blk_q && i < N;
        auto wait_all = [&](uint64_t *bar, uint32_t par) {
            const bool w = mbar_wait(bar, par, status, abort_flag);
            return __all_sync(0xffffffffu, w);
        };
        sm.mu[r] = __ldg(kmean + (size_t)bh * 128 + r);
        named_bar_sync(1, 128);
        const float c = kLog2e * kRsd;
        bool ok = true;
        // ---- pass 1: row max m, sum l and D = sum p dP (online, in log2 units; m is raised only when
        // the tile's max exceeds it by more than 2^8, so p stays below 256 and most tiles need no rescale)
        float m = -INFINITY, l = 0.0f, Dt = 0.0f;
        const uint64_t c2 = f2pack(c, c);
        int J_next = k_sel > 0 ? __ldg(sel) : 0;  // the selected blocks, loaded one tile ahead of use
        for (int t = 0; ok && t < k_sel; ++t) {
            const int T = t, b = T & 1;
            const int J = J_next, valid = min(64, N - J * 64);
            J_next = __ldg(sel + (t + 1 < k_sel ? t + 1 : 0));
            if (!(ok = wait_all(&sm.bar_sd[b], (T >> 1) & 1))) break;
            tc_fence_after();
            uint32_t sv[64], dv[64];
            tmem_ld64(tmem + 128 * b + lane_off, sv);
            tmem_ld64(tmem + 128 * b + 64 + lane_off, dv);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.bar_sdfree[b]);
            if (valid < 64) {  // the ragged last key block: its missing keys take no part
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (j >= valid) sv[j] = __float_as_uint(-INFINITY);
            }
            float tt[22];
#pragma unroll
            for (int j = 0; j < 21; ++j)
                tt[j] = fmax3f(__uint_as_float(sv[3 * j]), __uint_as_float(sv[3 * j + 1]), __uint_as_float(sv[3 * j + 2]));
            tt[21] = __uint_as_float(sv[63]);
#pragma unroll
            for (int j = 0; j < 7; ++j) tt[j] = fmax3f(tt[3 * j], tt[3 * j + 1], tt[3 * j + 2]);
            const float tmax =
                fmax3f(fmax3f(tt[0], tt[1], tt[2]), fmax3f(tt[3], tt[4], tt[5]), fmaxf(tt[6], tt[21])) * c;  // c > 0
            if (tmax > m + 8.0f) {  // also on the first tile (m = -inf)
                const float alpha = ex2f(m - tmax);  // 0 while m = -inf
                l *= alpha;
                Dt *= alpha;
                m = tmax;
            }
            const uint64_t nm2 = f2pack(-m, -m);
            uint64_t ls2 = 0, ds2 = 0;
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
                const float2 a = f2unpack(fma2(f2pack(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), c2, nm2));
                const uint64_t p2 = f2pack(ex2f(a.x), ex2f(a.y));  // masked keys: ex2(-inf) = 0
                ls2 = add2(ls2, p2);
                ds2 = fma2(p2, f2pack(__uint_as_float(dv[j]), __uint_as_float(dv[j + 1])), ds2);
            }
            const float2 ls = f2unpack(ls2), dsum = f2unpack(ds2);
            l += ls.x + ls.y;
            Dt += dsum.x + dsum.y;
        }
        const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
        const float D = Dt * inv_l;
        if (ok && row_valid) {
            st_m[(size_t)bh * N + i] = m;
            st_l[(size_t)bh * N + i] = inv_l;
            st_D[(size_t)bh * N + i] = D;
        }
        // ---- pass 2: dS (bf16) into shared memory for dQ += dS K
        float sigma = 0.0f;  // fp32 sum of the rounded dS of this row
        J_next = k_sel > 0 ? __ldg(sel) : 0;
        for (int t = 0; ok && t < k_sel; ++t) {
            const int T = k_sel + t, b = T & 1, bd = t & 1;
            const int J = J_next, valid = row_valid ? min(64, N - J * 64) : 0;
            J_next = __ldg(sel + (t + 1 < k_sel ? t + 1 : 0));
            if (!(ok = wait_all(&sm.bar_sd[b], (T >> 1) & 1))) break;
            tc_fence_after();
            uint32_t sv[64], dv[64];
            tmem_ld64(tmem + 128 * b + lane_off, sv);
            tmem_ld64(tmem + 128 * b + 64 + lane_off, dv);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.bar_sdfree[b]);
            if (valid < 64) {  // missing keys of the last block, and rows past the block: dS = 0
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (j >= valid) sv[j] = __float_as_uint(-INFINITY);
            }
            // dS = p (dP - D) / sqrt(d) with p = 2^(s c - m) / l, in packed pairs
            const uint64_t nm2 = f2pack(-m, -m), il2 = f2pack(inv_l * kRsd, inv_l * kRsd), nd2 = f2pack(-D, -D);
            uint32_t w[32];
            uint64_t sg2 = 0;
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
                const float2 a = f2unpack(fma2(f2pack(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), c2, nm2));
                const uint64_t p2 = mul2(f2pack(ex2f(a.x), ex2f(a.y)), il2);
                const float2 g = f2unpack(mul2(p2, add2(f2pack(__uint_as_float(dv[j]), __uint_as_float(dv[j + 1])), nd2)));
                w[j >> 1] = pack_bf16x2(g.x, g.y);
                sg2 = add2(sg2, f2pack(__uint_as_float(w[j >> 1] << 16), __uint_as_float(w[j >> 1] & 0xFFFF0000u)));
            }
            {
                const float2 sg = f2unpack(sg2);
                sigma += sg.x + sg.y;
            }
            if (t >= 2 && !(ok = wait_all(&sm.bar_dsfree[bd], ((t >> 1) - 1) & 1))) break;
            store_row_sw128(sm.ds[bd], r, w);
            fence_async_smem();
            mbar_arrive(&sm.bar_ds[bd]);
        }
        // ---- dq = dS K - sigma mu (zero without selected blocks)
        if (ok && k_sel > 0) ok = wait_all(&sm.bar_dq, 0);
        if (ok) {
            tc_fence_after();
            float *drow = dq + ((size_t)bh * N + (row_valid ? i : 0)) * 128;
#pragma unroll 1
            for (int c0 = 0; c0 < 128; c0 += 32) {
                uint32_t a[32];
                if (k_sel > 0) {
                    tmem_ld32(t_dq + lane_off + c0, a);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) a[e] = 0u;
                }
                if (row_valid) {
                    float4 *o = reinterpret_cast<float4 *>(drow + c0);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        o[e] = make_float4(fmaf(-sigma, sm.mu[c0 + 4 * e], __uint_as_float(a[4 * e])),
                                           fmaf(-sigma, sm.mu[c0 + 4 * e + 1], __uint_as_float(a[4 * e + 1])),
                                           fmaf(-sigma, sm.mu[c0 + 4 * e + 2], __uint_as_float(a[4 * e + 2])),
                                           fmaf(-sigma, sm.mu[c0 + 4 * e + 3], __uint_as_float(a[4 * e + 3])));
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

// ---------------------------------------------------------------------------
// key side
// ---------------------------------------------------------------------------
struct BkSmem {
    alignas(1024) uint8_t k[2 * kBox];               // K_J: ch 0-63 | 64-127
    alignas(1024) uint8_t v[2 * kBox];               // V_J: dims 0-63 | 64-127
    alignas(1024) uint8_t qd[kBkStages][4 * kTile];  // per stage: Q_I ch 0-63 | 64-127, dO_I dims 0-63 | 64-127
    alignas(1024) uint8_t p[2][kTile];               // P tiles: [128 query rows x 64 keys] bf16
    alignas(1024) uint8_t ds[2][kTile];              // dS tiles
    uint64_t full[kBkStages], empty[kBkStages];
    uint64_t bar_kv, bar_sd[2], bar_sdfree[2], bar_pd[2], bar_pdfree[2], bar_acc, drain;
    uint32_t tmem_base;
    int abort_flag;
};

// walks the set bits of a selection row (query blocks that selected a key block), in order
struct BitWalk {
    const uint32_t *bits;
    int words, w;
    uint32_t cur;
    SLA_DEV BitWalk(const uint32_t *b, int nw) : bits(b), words(nw), w(0), cur(nw > 0 ? __ldg(b) : 0u) {}
    SLA_DEV int next()
    {
        while (cur == 0u) {
            if (++w >= words) return -1;
            cur = __ldg(bits + w);
        }
        const int I = 32 * w + __ffs(cur) - 1;
        cur &= cur - 1u;
        return I;
    }
};

__global__ void __launch_bounds__(kBkThreads, 1)
bwdk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
            const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
            const uint32_t *__restrict__ selT, int n_awT, const float *__restrict__ st_m,
            const float *__restrict__ st_l, const float *__restrict__ st_D, int N, int blk_q, int n_qb, int n_kb,
            float *__restrict__ dk, float *__restrict__ dv, int *status)
{
    extern __shared__ uint8_t smem_raw[];
    BkSmem &sm = *reinterpret_cast<BkSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int J = blockIdx.x, bh = blockIdx.y;
    const int t0 = J * 64, kv = min(64, N - t0);
    const uint32_t *bits = selT + ((size_t)bh * n_kb + J) * n_awT;
    const int words = (n_qb + 31) / 32;
    int n_sel = 0;
    for (int w = 0; w < words; ++w) n_sel += __popc(__ldg(bits + w));
    volatile int *abort_flag = &sm.abort_flag;
    if (tid == 0) sm.abort_flag = global_failed(status) ? 1 : 0;
    __syncthreads();
    // no query block selected this key block (dk, dv hold the linear part alone), or another CTA
    // failed: CTA-uniform early exit
    if (sm.abort_flag || n_sel == 0) return;

    if (tid == 0) {
        for (int s = 0; s < kBkStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.bar_kv, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.bar_sd[b], 1);
            mbar_init(&sm.bar_sdfree[b], 256);
            mbar_init(&sm.bar_pd[b], 256);
            mbar_init(&sm.bar_pdfree[b], 1);
        }
        mbar_init(&sm.bar_acc, 1);
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;  // S / dP of buffer b at 128 b / 128 b + 64; dV^T at 256, dK^T at 320
    const uint32_t t_dv = tmem + 256, t_dk = tmem + 320;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (elect_one()) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_do);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_expect_tx(&sm.bar_kv, 4 * kBox);
            tma_load_4d(sm.k, &tm_k, &sm.bar_kv, 0, t0, 0, bh);
            tma_load_4d(sm.v, &tm_v, &sm.bar_kv, 0, t0, 0, bh);
        }
        __syncwarp();
        BitWalk walk(bits, words);
        int issued = 0;
        bool ok = true;
        for (int t = 0; ok && t < n_sel; ++t) {
            const int I = walk.next();
            const int s = t % kBkStages, u = t / kBkStages;
            if (u > 0 && !(ok = mbar_wait_warp(&sm.empty[s], (u - 1) & 1, status, abort_flag))) break;
            if (elect_one()) {
                mbar_expect_tx(&sm.full[s], 4 * kTile);
                tma_load_4d(sm.qd[s], &tm_q, &sm.full[s], 0, I * blk_q, 0, bh);
                tma_load_4d(sm.qd[s] + 2 * kTile, &tm_do, &sm.full[s], 0, I * blk_q, 0, bh);
            }
            __syncwarp();
            issued = t + 1;
        }
        for (int s = 0; s < kBkStages; ++s) {
            int tl = -1;
            for (int t = s; t < issued; t += kBkStages) tl = t;
            if (tl >= 0) mbar_wait_quiet(&sm.full[s], (tl / kBkStages) & 1, status);
        }
        mbar_wait_quiet(&sm.bar_kv, 0, status);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // dV^T += dO^T P and dK^T += Q^T dS: M = 128 dims / channels, N = 64 keys, K = 128 query rows,
        // A (dO, Q) and B (P, dS) both MN-major
        constexpr uint32_t id_acc = idesc(1, 1, 1, 1, 1, 128, 64);
        const uint64_t kd = sdesc_sw128(smem_u32(sm.k), 16, 1024), vd = sdesc_sw128(smem_u32(sm.v), 16, 1024);
        bool ok = mbar_wait_warp(&sm.bar_kv, 0, status, abort_flag);
        auto issue_sd = [&](int t) {
            const int s = t % kBkStages, b = t & 1;  // both phases were seen complete by the poll
            tc_fence_after();
            if (elect_one()) {
                issue_s_dp(tmem + 128 * b, tmem + 128 * b + 64, sdesc_sw128(smem_u32(sm.qd[s]), 16, 1024),
                           sdesc_sw128(smem_u32(sm.qd[s] + 2 * kTile), 16, 1024), kd, vd);
                mma_commit(&sm.bar_sd[b]);
            }
            __syncwarp();
        };
        auto issue_acc = [&](int t) {
            const int s = t % kBkStages, b = t & 1;  // the phase was seen complete by the poll
            tc_fence_after();
            if (elect_one()) {
                const uint64_t qmn = sdesc_sw128(smem_u32(sm.qd[s]), kTile, 1024);
                const uint64_t domn = sdesc_sw128(smem_u32(sm.qd[s] + 2 * kTile), kTile, 1024);
                const uint64_t pmn = sdesc_sw128(smem_u32(sm.p[b]), kTile, 1024);
                const uint64_t dsmn = sdesc_sw128(smem_u32(sm.ds[b]), kTile, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k) {  // K-step of 16 query rows: 2 KB of each tile; the chains alternate
                    mma_bf16(t_dv, dadd(domn, 2048 * k), dadd(pmn, 2048 * k), id_acc, (t > 0 || k > 0) ? 1u : 0u);
                    mma_bf16(t_dk, dadd(qmn, 2048 * k), dadd(dsmn, 2048 * k), id_acc, (t > 0 || k > 0) ? 1u : 0u);
                }
                mma_commit(&sm.bar_pdfree[b]);
                mma_commit(&sm.empty[s]);  // Q and dO of the stage are no longer read
                if (t == n_sel - 1) mma_commit(&sm.bar_acc);
            }
            __syncwarp();
        };
        // S/dP of tile t may run ahead of the accumulation of tile t-1 by one tile (two S/dP
        // buffers); between them, whichever is ready first is issued first: the accumulation frees
        // a Q/dO stage for the producer, S/dP feeds the row threads
        int n_sd = 0, n_acc = 0;
        long long t0c = clock64();
        const long long budget = wait_budget();
        while (ok && n_acc < n_sel) {
            const bool can_acc = n_acc < n_sd && mbar_test(&sm.bar_pd[n_acc & 1], (n_acc >> 1) & 1);
            if (__any_sync(0xffffffffu, can_acc)) {
                issue_acc(n_acc++);
                t0c = clock64();
                continue;
            }
            const bool can_sd = n_sd < n_sel && n_sd <= n_acc + 1 &&
                                mbar_test(&sm.full[n_sd % kBkStages], (n_sd / kBkStages) & 1) &&
                                (n_sd < 2 || mbar_test(&sm.bar_sdfree[n_sd & 1], ((n_sd >> 1) - 1) & 1));
            if (__any_sync(0xffffffffu, can_sd)) {
                issue_sd(n_sd++);
                t0c = clock64();
                continue;
            }
            if (clock64() - t0c > budget) {  // neither came: the same bounded-wait rule as mbar_wait
                if (elect_one()) record_error(status, kStatusTimeout);
                *abort_flag = 1;
                ok = false;
            } else if (global_failed(status) || *abort_flag) {
                *abort_flag = 1;
                ok = false;
            }
            ok = __all_sync(0xffffffffu, ok);
        }
        if (elect_one()) {
            mma_commit(&sm.drain);
            mbar_wait_quiet(&sm.drain, 0, status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ rows (query rows; dims at the end)
        // warps 2-5 take keys 0-31 of their rows, warps 6-9 keys 32-63
        const int quarter = warp & 3, half = (warp - 2) >> 2, j0 = 32 * half;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        auto wait_all = [&](uint64_t *bar, uint32_t par) {
            const bool w = mbar_wait(bar, par, status, abort_flag);
            return __all_sync(0xffffffffu, w);
        };
        const float c = kLog2e * kRsd;
        BitWalk walk(bits, words);
        bool ok = true;
        // this row's statistics in query block I (rows of the next query block when blk_q = 64, and
        // rows past N, take none); loaded one tile ahead of use
        auto stats = [&](int I, float &m, float &il, float &D) {
            const int i = I * blk_q + r;
            const bool rv = I >= 0 && r < blk_q && i < N;
            const size_t si = (size_t)bh * N + (rv ? i : 0);
            m = rv ? __ldg(st_m + si) : 0.0f;
            il = rv ? __ldg(st_l + si) : 0.0f;  // 0 for rows that take no part: P = 0
            D = rv ? __ldg(st_D + si) : 0.0f;
        };
        int I_next = walk.next();
        float m_n, il_n, D_n;
        stats(I_next, m_n, il_n, D_n);
        for (int t = 0; ok && t < n_sel; ++t) {
            const int I = I_next, b = t & 1;
            const float m = m_n, il = il_n, D = D_n;
            I_next = t + 1 < n_sel ? walk.next() : -1;
            stats(I_next, m_n, il_n, D_n);
            const int i = I * blk_q + r;
            const bool row_valid = r < blk_q && i < N;  // rows of the next query block (blk_q = 64) excluded
            const int valid = row_valid ? kv : 0;
            if (!(ok = wait_all(&sm.bar_sd[b], (t >> 1) & 1))) break;
            tc_fence_after();
            uint32_t sv[32], dpv[32];
            tmem_ld32(tmem + 128 * b + j0 + lane_off, sv);
            tmem_ld32(tmem + 128 * b + 64 + j0 + lane_off, dpv);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.bar_sdfree[b]);
            uint32_t wp[16], wd[16];
            if (valid < j0 + 32) {  // keys past the block's end (the ragged last block), or a row that takes no part
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j0 + j >= valid) sv[j] = __float_as_uint(-INFINITY);
            }
            const uint64_t c2 = f2pack(c, c), nm2 = f2pack(-m, -m), il2 = f2pack(il, il), nd2 = f2pack(-D, -D);
            const uint64_t rs2 = f2pack(kRsd, kRsd);
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                const float2 a = f2unpack(fma2(f2pack(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), c2, nm2));
                const uint64_t p2 = mul2(f2pack(ex2f(a.x), ex2f(a.y)), il2);
                const uint64_t g2 = mul2(mul2(p2, add2(f2pack(__uint_as_float(dpv[j]), __uint_as_float(dpv[j + 1])), nd2)), rs2);
                const float2 p = f2unpack(p2), g = f2unpack(g2);
                wp[j >> 1] = pack_bf16x2(p.x, p.y);
                wd[j >> 1] = pack_bf16x2(g.x, g.y);
            }
            if (t >= 2 && !(ok = wait_all(&sm.bar_pdfree[b], ((t >> 1) - 1) & 1))) break;
            // this thread's 64 bytes of row r: 16-byte units 4 half .. 4 half + 3
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                *reinterpret_cast<uint4 *>(sm.p[b] + sw128_off(r, 4 * half + u)) =
                    make_uint4(wp[4 * u], wp[4 * u + 1], wp[4 * u + 2], wp[4 * u + 3]);
                *reinterpret_cast<uint4 *>(sm.ds[b] + sw128_off(r, 4 * half + u)) =
                    make_uint4(wd[4 * u], wd[4 * u + 1], wd[4 * u + 2], wd[4 * u + 3]);
            }
            fence_async_smem();
            mbar_arrive(&sm.bar_pd[b]);
        }
        // ---- epilogue: TMEM lane r = dim / channel r; column j = key t0 + j.  Added to the linear part,
        // whose values are all loaded first (while the last accumulation runs), so that the 64
        // read-modify-writes of a thread do not wait on one another's loads
        float *pv = dv + ((size_t)bh * N + t0 + j0) * 128 + r;
        float *pk = dk + ((size_t)bh * N + t0 + j0) * 128 + r;
        float lv[32], lk[32];
        if (ok) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                lv[j] = j0 + j < kv ? __ldcg(pv + (size_t)j * 128) : 0.0f;
                lk[j] = j0 + j < kv ? __ldcg(pk + (size_t)j * 128) : 0.0f;
            }
            ok = wait_all(&sm.bar_acc, 0);
        }
        if (ok) {
            tc_fence_after();
            uint32_t a[32];
            tmem_ld32(t_dv + j0 + lane_off, a);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j0 + j < kv) pv[(size_t)j * 128] = lv[j] + __uint_as_float(a[j]);
            tmem_ld32(t_dk + j0 + lane_off, a);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j0 + j < kv) pk[(size_t)j * 128] = lk[j] + __uint_as_float(a[j]);
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

// ---------------------------------------------------------------------------
// linear branch.  Row i of query block I, f = phi(q_i), b = f . Z_I, a = f H_I,
// ol = a / b (zero when b = 0), da = do / b, db = -(do . ol) / b:
//   dq_i += (H_I da + Z_I db) phi'(q_i);  dH_I = sum_i f (outer) da;  dZ_I = sum_i f db;
// and for key block J, with G_J, g_J the sums of dH_I, dZ_I over the query blocks
// that did not select J:  dk_j = (G_J v_j + g_J) phi'(k_j);  dv_j = G_J^T phi(k_j).
// The d x d products run as bf16 tcgen05 MMAs with fp32 accumulation; the operand
// tiles are written by the threads in the 128-byte-swizzled layout, [rows x 128 B]
// boxes of 64 bf16 (two boxes per 128 columns).
//
// Centring.  When the values share a common component, H_I da and Z_I db nearly
// cancel in dq (H_I ~ Z_I (outer) mean value), and so do G_J v_j and g_J in dk; bf16
// operands would then carry errors relative to the large terms.  Both sides are
// therefore evaluated with centred operands, which is exact algebra: for any vector
// mu, with H' = H_I - Z_I (outer) mu, a' = f H', ol = a' / b + mu, and
//   H_I da + Z_I db = H' da + Z_I db',  db' = -(da . a') / b,  db = db' - da . mu;
// the kernel takes mu_e = (sum_c Z_c H[c][e]) / (sum_c Z_c^2), the least-squares fit
// of H_I by Z_I (outer) mu, and rounds H' to bf16 (dZ_I still uses the true db).  On
// the key side, with nu the key block's mean value row,
//   G_J v_j + g_J = G_J (v_j - nu) + (g_J + G_J nu),
// where the second term is summed in fp32.
// ---------------------------------------------------------------------------
constexpr int kLinThreads = 128;

SLA_DEV float phi_lin(float x, int phi)
{
    if (phi == 1) return fmaxf(x, 0.0f);
    const float e = ex2f(fminf(x, 0.0f) * kLog2e);
    return x > 0.0f ? x + 1.0f : e;
}

SLA_DEV float dphi_lin(float x, int phi)
{
    if (phi == 1) return x > 0.0f ? 1.0f : 0.0f;
    const float e = ex2f(fminf(x, 0.0f) * kLog2e);
    return x > 0.0f ? 1.0f : e;
}

// row r of a [rows x 128 bf16] operand (two [rows x 128 B] boxes `box` bytes apart): element c = val(c)
template <class F>
SLA_DEV void store_row128(uint8_t *tile, uint32_t box, int r, F val)
{
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] = pack_bf16x2(val(64 * h + 2 * e), val(64 * h + 2 * e + 1));
        store_row_sw128(tile + h * box, r, w);
    }
}

// element (r, c) of a [rows x 128 bf16] operand written by store_row128
SLA_DEV float load_elem128(const uint8_t *tile, uint32_t box, int r, int c)
{
    const uint16_t *p = reinterpret_cast<const uint16_t *>(tile + (c >> 6) * box + sw128_off(r, (c & 63) >> 3)) + (c & 7);
    return __uint_as_float((uint32_t)*p << 16);
}

struct LqSmem {
    alignas(1024) uint8_t hs[4 * kTile];  // H_I^T fp32: four [128 dims x 32 channels] tiles; later dq staging
    alignas(1024) uint8_t qr[2 * kTile];  // raw Q rows of the query block (bf16, [rows x 64 channels] boxes)
    alignas(1024) uint8_t da[2 * kTile];  // dO rows as loaded, then dA in place ([row i][dim e]: K-major A of H da,
                                          // MN-major B of dH)
    alignas(1024) uint8_t f[2 * kTile];   // F = phi(Q_I) [row i][channel c] (K-major A of a; MN-major A of dH)
    alignas(1024) uint8_t h[2 * kTile];   // centred H'^T [dim e][channel c] (K-major B of a; MN-major B of H da)
    float z[128], db[128], mu[128];
    uint64_t bar_ld, bar_a, bar_d;
    uint32_t tmem_base;
};

// byte offset of fp32 element c of row r in a tile of four [rows x 32 fp32] boxes with the 128-byte swizzle
SLA_DEV uint32_t f32_off(int r, int c) { return (c >> 5) * kTile + sw128_off(r, (c & 31) >> 2) + (c & 3) * 4; }

// query side: dq (added to the softmax branch's), dH_I and dZ_I (fp32 and bf16).  Every operand arrives by
// TMA (H_I, the Q and dO rows); the dq update goes through shared memory so that its global accesses are
// whole coalesced rows.
__global__ void __launch_bounds__(kLinThreads, 1)
bwd_qlin_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_do, const float *__restrict__ hq, int N, int blk_q, int n_qb,
                int phi, float *__restrict__ dq, float *__restrict__ dh32, uint16_t *__restrict__ dh16, int *status)
{
    extern __shared__ uint8_t smem_raw[];
    LqSmem &sm = *reinterpret_cast<LqSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int I = blockIdx.x, bh = blockIdx.y;
    const int r = tid;
    const int rows = min(blk_q, N - I * blk_q);
    const bool row_valid = r < rows;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    if (tid == 0) {
        mbar_init(&sm.bar_ld, 1);
        mbar_init(&sm.bar_a, 1);
        mbar_init(&sm.bar_d, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        mbar_expect_tx(&sm.bar_ld, 8 * kTile);
        tma_load_4d(sm.hs, &tm_h, &sm.bar_ld, 0, 0, 0, bh * n_qb + I);
        tma_load_4d(sm.qr, &tm_q, &sm.bar_ld, 0, I * blk_q, 0, bh);
        tma_load_4d(sm.da, &tm_do, &sm.bar_ld, 0, I * blk_q, 0, bh);
    }
    const float *hrow = hq + ((size_t)bh * n_qb + I) * kStateCols;
    sm.z[tid] = __ldg(hrow + 128 * 128 + tid);
    bool ok = __all_sync(0xffffffffu, mbar_wait_quiet(&sm.bar_ld, 0, status));
    __syncthreads();  // z visible
    const uint32_t tmem = sm.tmem_base, t_a = tmem, t_d = tmem + 128;  // a then dH at 0; dF at 128
    // ---- row e = tid of the centred H'^T = H_I^T - mu (outer) Z_I
    {
        const int e = tid;
        float zh = 0.0f, zz = 0.0f;
#pragma unroll 8
        for (int u = 0; u < 32; ++u) {
            const float4 h = *reinterpret_cast<const float4 *>(sm.hs + f32_off(e, 4 * u));
            zh = fmaf(sm.z[4 * u], h.x, fmaf(sm.z[4 * u + 1], h.y, fmaf(sm.z[4 * u + 2], h.z, fmaf(sm.z[4 * u + 3], h.w, zh))));
            zz = fmaf(sm.z[4 * u], sm.z[4 * u], fmaf(sm.z[4 * u + 1], sm.z[4 * u + 1],
                      fmaf(sm.z[4 * u + 2], sm.z[4 * u + 2], fmaf(sm.z[4 * u + 3], sm.z[4 * u + 3], zz))));
        }
        const float mu = zz > 0.0f ? zh / zz : 0.0f;
        sm.mu[e] = mu;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t w[32];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int c = 64 * hh + 4 * u;
                const float4 h = *reinterpret_cast<const float4 *>(sm.hs + f32_off(e, c));
                w[2 * u] = pack_bf16x2(fmaf(-mu, sm.z[c], h.x), fmaf(-mu, sm.z[c + 1], h.y));
                w[2 * u + 1] = pack_bf16x2(fmaf(-mu, sm.z[c + 2], h.z), fmaf(-mu, sm.z[c + 3], h.w));
            }
            store_row_sw128(sm.h + hh * kTile, e, w);
        }
    }
    // 8 bf16 channels 8u .. 8u + 7 of row r of a [rows x 128 bf16] tile (two [rows x 64] boxes)
    auto unit8 = [&](const uint8_t *tile, int u, float (&x)[8]) {
        const uint4 w = *reinterpret_cast<const uint4 *>(tile + (u >> 3) * kTile + sw128_off(r, u & 7));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[2 * e] = __uint_as_float(ww[e] << 16);
            x[2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
        }
    };
    // ---- F row (zero past the block's rows) and b = f . Z_I
    float b = 0.0f;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        uint32_t w[32];
#pragma unroll
        for (int uu = 0; uu < 8; ++uu) {
            float x[8];
            unit8(sm.qr, 8 * hh + uu, x);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                x[e] = row_valid ? phi_lin(x[e], phi) : 0.0f;
                b = fmaf(x[e], sm.z[64 * hh + 8 * uu + e], b);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) w[4 * uu + e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
        }
        store_row_sw128(sm.f + hh * kTile, r, w);
    }
    const float binv = (row_valid && b != 0.0f) ? 1.0f / b : 0.0f;
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // a' = F H': M = 128 rows, N = 128 dims, K = 128 channels
    if (tid == 0 && ok) {
        constexpr uint32_t id = idesc(1, 1, 1, 0, 0, 128, 128);
        const uint64_t fd = sdesc_sw128(smem_u32(sm.f), 16, 1024), hd = sdesc_sw128(smem_u32(sm.h), 16, 1024);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * kTile + (k & 3) * 32;
            mma_bf16(t_a, dadd(fd, off), dadd(hd, off), id, k > 0 ? 1u : 0u);
        }
        mma_commit(&sm.bar_a);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_quiet(&sm.bar_a, 0, status));
    // ---- db' = -(do . a') / b^2, dA = do / b (in place of the dO row), and the true db = db' - da . mu
    float db = 0.0f;
    if (ok) {
        tc_fence_after();
        float dot = 0.0f, dmu = 0.0f;
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t a[32];
            tmem_ld32(t_a + lane_off + c0, a);
            tmem_wait_ld();
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
                float x[8];
                unit8(sm.da, (c0 >> 3) + uu, x);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    dot = fmaf(x[e], __uint_as_float(a[8 * uu + e]), dot);
                    dmu = fmaf(x[e], sm.mu[c0 + 8 * uu + e], dmu);
                }
            }
        }
        db = -(dot * binv) * binv;  // db' of the centred state
        sm.db[tid] = db - dmu * binv;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t w[32];
#pragma unroll
            for (int uu = 0; uu < 8; ++uu) {
                float x[8];
                unit8(sm.da, 8 * hh + uu, x);
#pragma unroll
                for (int e = 0; e < 4; ++e) w[4 * uu + e] = pack_bf16x2(x[2 * e] * binv, x[2 * e + 1] * binv);
            }
            store_row_sw128(sm.da + hh * kTile, r, w);
        }
    } else {
        sm.db[tid] = 0.0f;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // dF = dA H'^T (N = 128 channels: H'^T as an MN-major B) and dH = F^T dA (M = 128 channels,
    // N = 128 dims, K = 128 rows: both operands MN-major), into the dF and a columns
    if (tid == 0 && ok) {
        constexpr uint32_t id_df = idesc(1, 1, 1, 0, 1, 128, 128), id_dh = idesc(1, 1, 1, 1, 1, 128, 128);
        const uint64_t dad = sdesc_sw128(smem_u32(sm.da), 16, 1024);
        const uint64_t hmn = sdesc_sw128(smem_u32(sm.h), kTile, 1024);
        const uint64_t fmn = sdesc_sw128(smem_u32(sm.f), kTile, 1024), damn = sdesc_sw128(smem_u32(sm.da), kTile, 1024);
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // K-step of 16: the two chains alternate
            mma_bf16(t_d, dadd(dad, (k >> 2) * kTile + (k & 3) * 32), dadd(hmn, 2048 * k), id_df, k > 0 ? 1u : 0u);
            mma_bf16(t_a, dadd(fmn, 2048 * k), dadd(damn, 2048 * k), id_dh, k > 0 ? 1u : 0u);
        }
        mma_commit(&sm.bar_d);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_quiet(&sm.bar_d, 0, status));
    if (ok) {
        tc_fence_after();
        // dq row delta (dF + Z_I db') phi'(q) into the staging tile (the H_I^T region is free now)
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t a[32];
            tmem_ld32(t_d + lane_off + c0, a);
            tmem_wait_ld();
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
                float x[8];
                unit8(sm.qr, (c0 >> 3) + uu, x);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int e = 8 * uu + 4 * hh, c = c0 + e;
                    *reinterpret_cast<float4 *>(sm.hs + f32_off(r, c)) = make_float4(
                        fmaf(sm.z[c], db, __uint_as_float(a[e])) * dphi_lin(x[4 * hh], phi),
                        fmaf(sm.z[c + 1], db, __uint_as_float(a[e + 1])) * dphi_lin(x[4 * hh + 1], phi),
                        fmaf(sm.z[c + 2], db, __uint_as_float(a[e + 2])) * dphi_lin(x[4 * hh + 2], phi),
                        fmaf(sm.z[c + 3], db, __uint_as_float(a[e + 3])) * dphi_lin(x[4 * hh + 3], phi));
                }
            }
        }
        // dH (TMEM lane = channel c = tid, column = dim e) stored as dH^T [e][c]
        float *d32 = dh32 + ((size_t)bh * n_qb + I) * kStateCols;
        uint16_t *d16 = dh16 + ((size_t)bh * n_qb + I) * kStateCols;
        const int c = tid;
#pragma unroll 1
        for (int e0 = 0; e0 < 128; e0 += 32) {
            uint32_t a[32];
            tmem_ld32(t_a + lane_off + e0, a);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float x = __uint_as_float(a[e]);
                d32[(size_t)(e0 + e) * 128 + c] = x;
                d16[(size_t)(e0 + e) * 128 + c] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
            }
        }
        // dZ_I[c] = sum_i F[i][c] db_i
        float dz = 0.0f;
        for (int rr = 0; rr < 128; ++rr) dz = fmaf(load_elem128(sm.f, kTile, rr, c), sm.db[rr], dz);
        d32[128 * 128 + c] = dz;
        d16[128 * 128 + c] = __bfloat16_as_ushort(__float2bfloat16_rn(dz));
    }
    __syncthreads();  // the dq deltas are staged
    if (ok) {
        // dq += the staged deltas: warp w takes rows 32 w .. 32 w + 31, one coalesced 512-byte row per
        // step, eight rows' loads issued before their stores
#pragma unroll 1
        for (int r0 = 0; r0 < 32; r0 += 8) {
            float4 v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int row = warp * 32 + r0 + q;
                if (row < rows)
                    v[q] = __ldcg(reinterpret_cast<const float4 *>(dq + ((size_t)bh * N + I * blk_q + row) * 128) + lane);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int row = warp * 32 + r0 + q;
                if (row < rows) {
                    const float4 d = *reinterpret_cast<const float4 *>(sm.hs + f32_off(row, 4 * lane));
                    v[q].x += d.x; v[q].y += d.y; v[q].z += d.z; v[q].w += d.w;
                    reinterpret_cast<float4 *>(dq + ((size_t)bh * N + I * blk_q + row) * 128)[lane] = v[q];
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

struct LkSmem {
    alignas(1024) uint8_t g[2 * kTile];   // G_J^T as [dim e][channel c] bf16 (MN-major A of G v; K-major A of G^T phi(k))
    alignas(1024) uint8_t v[2 * kBox];    // V_J - nu as [key j][dim e] (K-major B of G v)
    alignas(1024) uint8_t fk[2 * kBox];   // phi(K_J) as [key j][channel c] (K-major B of G^T phi(k))
    float gz[128], nu[128], gp[128];      // g_J, the block's mean value row nu, g_J + G_J nu
    uint64_t bar;
    uint32_t tmem_base;
};

// key side: dk, dv of the linear branch, written (the softmax branch's key side adds to them)
__global__ void __launch_bounds__(kLinThreads, 3)
bwd_klin_kernel(const uint16_t *__restrict__ k, const uint16_t *__restrict__ v, const float *__restrict__ G, int N,
                int n_kb, int phi, float *__restrict__ dk, float *__restrict__ dv, int *status)
{
    extern __shared__ uint8_t smem_raw[];
    LkSmem &sm = *reinterpret_cast<LkSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int J = blockIdx.x, bh = blockIdx.y;
    const int t0 = J * 64, kv = min(64, N - t0);
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    if (tid == 0) {
        mbar_init(&sm.bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 128);
        tmem_relinquish();
    }
    const float *grow = G + ((size_t)bh * n_kb + J) * kStateCols;
    {
        // G_J^T rows e: each warp takes 32, one coalesced 512-byte row per load (lane: 4 channels)
        const int lane = tid & 31, c0 = 4 * lane;
#pragma unroll 4
        for (int rr = 0; rr < 32; ++rr) {
            const int e = warp * 32 + rr;
            const float4 g = __ldg(reinterpret_cast<const float4 *>(grow + (size_t)e * 128) + lane);
            uint2 *dst = reinterpret_cast<uint2 *>(sm.g + (c0 >> 6) * kTile + sw128_off(e, (c0 & 63) >> 3) + (c0 & 7) * 2);
            *dst = make_uint2(pack_bf16x2(g.x, g.y), pack_bf16x2(g.z, g.w));
        }
    }
    sm.gz[tid] = __ldg(grow + 128 * 128 + tid);
    // nu = the block's mean value row (dims e = tid), in fp32 from the bf16 rows (the loads are issued
    // together: a fixed trip count, predicated)
    {
        const int e = tid;
        const uint16_t *ve = v + ((size_t)bh * N + t0) * 128 + e;
        float sv[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < 64; ++j)
            if (j < kv) sv[j & 7] += __uint_as_float((uint32_t)__ldg(ve + (size_t)j * 128) << 16);
        sm.nu[e] = (((sv[0] + sv[1]) + (sv[2] + sv[3])) + ((sv[4] + sv[5]) + (sv[6] + sv[7]))) / (float)kv;
    }
    __syncthreads();
    {
        // thread -> (key row j = tid % 64, half h = tid / 64 of its 128 columns): V - nu and phi(K) rows
        const int j = tid & 63, h = tid >> 6;
        const bool ok = j < kv;
        const uint4 *vs = reinterpret_cast<const uint4 *>(v + ((size_t)bh * N + t0 + (ok ? j : 0)) * 128 + 64 * h);
        const uint4 *ks = reinterpret_cast<const uint4 *>(k + ((size_t)bh * N + t0 + (ok ? j : 0)) * 128 + 64 * h);
        uint32_t wv[32], wk[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint4 a = ok ? __ldg(vs + u) : make_uint4(0, 0, 0, 0);
            const uint4 c = ok ? __ldg(ks + u) : make_uint4(0, 0, 0, 0);
            const uint32_t aa[4] = {a.x, a.y, a.z, a.w}, cc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d0 = 64 * h + 8 * u + 2 * e;
                const float vlo = ok ? __uint_as_float(aa[e] << 16) - sm.nu[d0] : 0.0f;
                const float vhi = ok ? __uint_as_float(aa[e] & 0xFFFF0000u) - sm.nu[d0 + 1] : 0.0f;
                wv[4 * u + e] = pack_bf16x2(vlo, vhi);
                const float lo = ok ? phi_lin(__uint_as_float(cc[e] << 16), phi) : 0.0f;
                const float hi = ok ? phi_lin(__uint_as_float(cc[e] & 0xFFFF0000u), phi) : 0.0f;
                wk[4 * u + e] = pack_bf16x2(lo, hi);
            }
        }
        store_row_sw128(sm.v + h * kBox, j, wv);
        store_row_sw128(sm.fk + h * kBox, j, wk);
    }
    // g' = g_J + G_J nu (fp32): channel c = tid, G_J[c][e] = G_J^T[e][c] (coalesced across the warp)
    {
        const int c = tid;
        float gg[4] = {sm.gz[c], 0.0f, 0.0f, 0.0f};
#pragma unroll 32
        for (int e = 0; e < 128; ++e) gg[e & 3] = fmaf(__ldg(grow + (size_t)e * 128 + c), sm.nu[e], gg[e & 3]);
        sm.gp[c] = (gg[0] + gg[1]) + (gg[2] + gg[3]);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base, t_k = tmem, t_v = tmem + 64;
    if (tid == 0) {
        // T^T = G V^T: M = 128 channels, N = 64 keys, K = 128 dims (A = G_J^T tile read MN-major);
        // dV^T = G^T phi(K)^T: M = 128 dims, N = 64 keys, K = 128 channels (A K-major)
        constexpr uint32_t id_k = idesc(1, 1, 1, 1, 0, 128, 64), id_v = idesc(1, 1, 1, 0, 0, 128, 64);
        const uint64_t gmn = sdesc_sw128(smem_u32(sm.g), kTile, 1024), gk = sdesc_sw128(smem_u32(sm.g), 16, 1024);
        const uint64_t vd = sdesc_sw128(smem_u32(sm.v), 16, 1024), fd = sdesc_sw128(smem_u32(sm.fk), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            mma_bf16(t_k, dadd(gmn, 2048 * kk), dadd(vd, (kk >> 2) * kBox + (kk & 3) * 32), id_k, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            mma_bf16(t_v, dadd(gk, (kk >> 2) * kTile + (kk & 3) * 32), dadd(fd, (kk >> 2) * kBox + (kk & 3) * 32), id_v,
                     kk > 0 ? 1u : 0u);
        mma_commit(&sm.bar);
    }
    const bool ok = __all_sync(0xffffffffu, mbar_wait_quiet(&sm.bar, 0, status));
    if (ok) {
        tc_fence_after();
        const int c = tid;  // TMEM lane: channel c (dk) and dim c (dv)
        uint32_t a[64];
        tmem_ld64(t_k + lane_off, a);
        tmem_wait_ld();
        const size_t base = ((size_t)bh * N + t0) * 128 + c;
#pragma unroll
        for (int j0 = 0; j0 < 64; j0 += 32) {  // 32 keys' loads issued before their stores
            uint16_t kb[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) kb[j] = j0 + j < kv ? __ldg(k + base + (size_t)(j0 + j) * 128) : (uint16_t)0;
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j0 + j < kv)
                    dk[base + (size_t)(j0 + j) * 128] =
                        (__uint_as_float(a[j0 + j]) + sm.gp[c]) * dphi_lin(__uint_as_float((uint32_t)kb[j] << 16), phi);
        }
        tmem_ld64(t_v + lane_off, a);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 64; ++j)
            if (j < kv) dv[base + (size_t)j * 128] = __uint_as_float(a[j]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// Map of a bf16 tensor [BH, N, 128] viewed as [64 elements, N rows (256 B apart), 2 halves (128 B
// apart), BH]: one box of {64, rows, 2, 1} lands as the two [rows x 128 B] half-tiles (channels 0-63,
// then 64-127) one after the other.  One copy per tile instead of two: a copy costs the issuing CTA
// about the same whatever its size.
bool map_rows(CUtensorMap *m, const void *base, const Geometry &g, uint32_t rows)
{
    const uint64_t dims[4] = {64, (uint64_t)g.N, 2, (uint64_t)g.BH};
    const uint64_t st[3] = {(uint64_t)kD * 2, 128, (uint64_t)g.N * kD * 2};
    const uint32_t box[4] = {64, rows, 2, 1};
    return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, st, box);
}

}  // namespace

cudaError_t launch_bwd_query_sparse(const void *q, const void *k, const void *v, const void *dout,
                                    const int32_t *idx, const float *kmean, const Geometry &g, float *dq,
                                    float *st_m, float *st_l, float *st_D, int *status, cudaStream_t s)
{
    CUtensorMap tq, tdo, tk, tv;
    if (!map_rows(&tq, q, g, 128) || !map_rows(&tdo, dout, g, 128) || !map_rows(&tk, k, g, 64) ||
        !map_rows(&tv, v, g, 64))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(BqSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(bwdq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwdq_kernel<<<dim3(g.n_qb, g.BH), kBwThreads, smem, s>>>(tq, tdo, tk, tv, idx, kmean, g.N, g.blk_q, g.n_qb,
                                                             g.k_sel, dq, st_m, st_l, st_D, status);
    return cudaGetLastError();
}

cudaError_t launch_bwd_key_sparse(const void *q, const void *k, const void *v, const void *dout,
                                  const uint32_t *selT, int n_awT, const float *st_m, const float *st_l,
                                  const float *st_D, const Geometry &g, float *dk, float *dv, int *status,
                                  cudaStream_t s)
{
    CUtensorMap tq, tdo, tk, tv;
    if (!map_rows(&tq, q, g, 128) || !map_rows(&tdo, dout, g, 128) || !map_rows(&tk, k, g, 64) ||
        !map_rows(&tv, v, g, 64))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(BkSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(bwdk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwdk_kernel<<<dim3(g.n_kb, g.BH), kBkThreads, smem, s>>>(tq, tdo, tk, tv, selT, n_awT, st_m, st_l, st_D, g.N,
                                                             g.blk_q, g.n_qb, g.n_kb, dk, dv, status);
    return cudaGetLastError();
}

cudaError_t launch_bwd_query_linear(const void *q, const void *dout, const float *hq, const Geometry &g, int phi,
                                    float *dq, float *dh32, uint16_t *dh16, int *status, cudaStream_t s)
{
    CUtensorMap th, tq, tdo;
    {
        // H_I^T of every query block: [BH * n_qb][128 dims][128 channels] fp32 inside rows of kStateCols,
        // viewed as [32 channels, 128 dims (512 B apart), 4 quarters (128 B apart), BH * n_qb]: one box
        // lands as the four [128 x 128 B] quarter-tiles one after the other
        const uint64_t hd[4] = {32, (uint64_t)kD, 4, (uint64_t)g.BH * g.n_qb};
        const uint64_t st[3] = {(uint64_t)kD * 4, 128, (uint64_t)kStateCols * 4};
        const uint32_t bx[4] = {32, 128, 4, 1};
        if (!encode_tmap(&th, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, hq, hd, st, bx)) return cudaErrorInvalidValue;
    }
    if (!map_rows(&tq, q, g, 128) || !map_rows(&tdo, dout, g, 128)) return cudaErrorInvalidValue;
    const size_t smem = sizeof(LqSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(bwd_qlin_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_qlin_kernel<<<dim3(g.n_qb, g.BH), kLinThreads, smem, s>>>(th, tq, tdo, hq, g.N, g.blk_q, g.n_qb, phi, dq, dh32,
                                                                  dh16, status);
    return cudaGetLastError();
}

cudaError_t launch_bwd_key_linear(const void *k, const void *v, const float *G, const Geometry &g, int phi, float *dk,
                                  float *dv, int *status, cudaStream_t s)
{
    const size_t smem = sizeof(LkSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(bwd_klin_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_klin_kernel<<<dim3(g.n_kb, g.BH), kLinThreads, smem, s>>>(static_cast<const uint16_t *>(k),
                                                                  static_cast<const uint16_t *>(v), G, g.N, g.n_kb,
                                                                  phi, dk, dv, status);
    return cudaGetLastError();
}

cudaError_t set_wait_budget_bwd(long long cycles) { return set_tu_wait_budget(cycles); }

}  // namespace sla
