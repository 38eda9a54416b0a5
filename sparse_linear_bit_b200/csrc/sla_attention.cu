// sla_attention.cu -- fused block-sparse attention + linear epilogue of the
// SageSLA forward (one CTA per (batch*head, query block)).
//
// Sparse branch: exact softmax attention softmax(q k^T / sqrt(d)) v
// ("TurboDiffusion技术架构解析" §2.1, standard attention formula) over the tokens
// of the key blocks the query block selected, computed SageAttention-style
// ("清华开源TurboDiffusion加速框架", SageAttention与稀疏计算): INT8 Q.K^T on the
// tensor cores with per-block fp32 dequantisation scales (or FP8 e4m3 codes
// on the f8f6f4 tensor-core path with fp32 sums), online softmax in fp32, P
// rounded to bf16 for a bf16 P.V with fp32 accumulation.  With
// quantisation off, Q.K^T runs in bf16 and P.V in fp16 (P and an fp16 copy of
// V, 8x finer rounding than bf16), both with fp32 accumulation.
//
// Linear branch epilogue: phi(Q_I) H_I as a tf32 MMA into its own TMEM
// accumulator, normalised by phi(q) . Z_I on the CUDA cores; output =
// sparse + linear, rounded to bf16.
//
// Tiling.  Key blocks are processed in selection order, loaded two per ring
// stage.  Two softmax warpgroups take one block each (warpgroup g: blocks
// 2t+g) with their own S (one M=128, N=64 Q.K^T chain per block), P, O
// accumulator and running (max, sum), merged in the epilogue; the groups share
// nothing but Q, the ring and the exponential token, so one group's Q.K^T is
// issued while the other group is still reading its logits.  The two
// warps that share an SM sub-partition (same query rows, one per group) pass a
// token so that their exponential phases alternate: the MUFU unit is the
// scarcest resource, and one group's exponentials overlap the other group's
// TMEM loads, row maxima and stores.
//
// Issue.  tcgen05 and mbarrier operations cost tens of cycles each on the
// issuing thread, so each softmax group has its own issuing thread for its
// Q.K^T and P.V.  Dependencies go through mbarriers only: S of a group is
// rewritten once that group has read it; P of a group is rewritten once that
// group's previous P.V has completed.
//
// Shared-memory bandwidth (128 B/clk, shared by TMA writes and tensor-core
// operand reads): both A operands live in tensor memory -- Q (written once per
// CTA from registers) and P (packed two 16-bit values per 32-bit column) -- so
// per key block only K and V cross shared memory, through a ring of four
// pair-stages.  The linear branch runs at the end, reusing the ring for its
// operands and the S columns for its accumulator.
//
// Roles (384 threads): warp 0 TMA producer, warp 1 linear-branch issuer and
// TMEM owner, warps 2-5 / 6-9 softmax groups 0 / 1 (one query row per thread,
// one TMEM lane quarter per warp), warps 10 / 11 Q.K^T + P.V issuers of groups
// 0 / 1.  TMEM columns: S of group g at 64g (L over both at the end), P of
// group g at 128 + 32g, Q at 192, O of group g at 256 + 128g.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "sla_internal.h"
#include "sla_ptx.cuh"

namespace sla {
namespace {

constexpr int kAttnThreads = 384;
constexpr uint32_t kBox = 64 * 128;          // [64 rows x 128 B]
constexpr uint32_t kQRowsBox = 128 * 128;    // [128 rows x 128 B]
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;    // log2 units: P may grow to 2^8 before O is rescaled
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1 / sqrt(128)

template <bool QUANT>  // QUANT: 8-bit Q/K codes (INT8 or FP8)
struct AttnCfg {
    static constexpr uint32_t kKBytes = QUANT ? 2 * kBox : 4 * kBox;        // K of a pair of key blocks
    static constexpr uint32_t kVBytes = 4 * kBox;                           // V of a pair of key blocks
    static constexpr uint32_t kStageBytes = kKBytes + kVBytes;
    static constexpr int kStages = QUANT ? 4 : 3;
    static constexpr uint32_t kLinBytes = 10 * kQRowsBox;  // H_I 64 KB + phi(Q) 64 KB + raw Q 32 KB
    static constexpr uint32_t kRegion = (kStages * kStageBytes > kLinBytes) ? kStages * kStageBytes : kLinBytes;
};

template <bool QUANT>
struct AttnSmem {
    alignas(1024) uint8_t region[AttnCfg<QUANT>::kRegion];  // K/V ring, then the linear operands
    float z[kD];
    float fin[2][3][128];   // epilogue exchange: [group][max, sum, den]
    uint64_t bar_q, bar_h, bar_qr, bar_phiq, bar_lin, drain[3];
    uint64_t full[AttnCfg<QUANT>::kStages], empty[AttnCfg<QUANT>::kStages];
    uint64_t bar_s[2], bar_sfree[2], bar_p[2], bar_pv[2];
    uint64_t tok[2][4];     // exponential-phase token per group and lane quarter
    uint32_t tmem_base;
    int abort_flag;
};

SLA_DEV float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// phi of one Q element, rounded to tf32 for the linear branch's MMA.  exp(x) for
// x <= 0 is ex2(x log2 e) on the MUFU unit (the result is rounded to 10 mantissa
// bits next).
SLA_DEV float phi_tf32(float x, int phi)
{
    const float e = ex2(fminf(x, 0.0f) * kLog2e);  // unconditional, so both cases are a select
    return to_tf32(phi == 1 ? fmaxf(x, 0.0f) : (x > 0.0f ? x + 1.0f : e));
}

SLA_DEV void named_bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// A from tensor memory (rows = lanes, two 16-bit K elements per 32-bit column)
SLA_DEV void mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc_, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc_), "r"(accumulate)
        : "memory");
}

// Row max over this thread's 64 tile columns, in logit units (log2 domain).
// INT_S: raw int32 dot products; adding the 1.5 * 2^23 bias to the bits makes them
// floats 12582912 + d (exact for |d| < 2^22), which is also how tile_exp reads them.
// Otherwise the logits are fp32 already.
template <bool INT_S, bool MASKED>
SLA_DEV float tile_max(uint32_t (&sv)[64], int valid, float c)
{
    if (INT_S) {
#pragma unroll
        for (int k = 0; k < 64; ++k) sv[k] += 0x4B400000u;
    }
    if (MASKED) {
        if (valid == 0) return -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; ++k)
            if (k >= valid) sv[k] = __float_as_uint(-INFINITY);
    }
    float tt[22];
#pragma unroll
    for (int k = 0; k < 21; ++k)
        tt[k] = fmax3f(__uint_as_float(sv[3 * k]), __uint_as_float(sv[3 * k + 1]), __uint_as_float(sv[3 * k + 2]));
    tt[21] = __uint_as_float(sv[63]);
#pragma unroll
    for (int k = 0; k < 7; ++k) tt[k] = fmax3f(tt[3 * k], tt[3 * k + 1], tt[3 * k + 2]);
    const float xmax = fmax3f(fmax3f(tt[0], tt[1], tt[2]), fmax3f(tt[3], tt[4], tt[5]), fmaxf(tt[6], tt[21]));
    return (INT_S ? (xmax - 12582912.0f) : xmax) * c;  // c >= 0
}

// P = exp2(x * c + off) for the 64 columns, packed two per 32-bit word; returns the row sum.
template <bool P_BF16, bool MASKED>
SLA_DEV float tile_exp(const uint32_t (&sv)[64], int valid, float c, float off, uint32_t (&pk)[32])
{
    const uint64_t c2 = f2pack(c, c), off2 = f2pack(off, off);
    uint64_t acc2[4] = {0, 0, 0, 0};
#pragma unroll
    for (int k = 0; k < 64; k += 2) {
        const float2 arg = f2unpack(fma2(f2pack(__uint_as_float(sv[k]), __uint_as_float(sv[k + 1])), c2, off2));
        float p0 = ex2(arg.x), p1 = ex2(arg.y);
        if (MASKED) {  // masked columns: P = 0 exactly (even when c = 0)
            if (k >= valid) p0 = 0.0f;
            if (k + 1 >= valid) p1 = 0.0f;
        }
        acc2[(k >> 1) & 3] = add2(acc2[(k >> 1) & 3], f2pack(p0, p1));
        pk[k >> 1] = P_BF16 ? pack_bf16x2(p0, p1) : pack_f16x2_sat(p0, p1);
    }
    const float2 s01 = f2unpack(add2(add2(acc2[0], acc2[1]), add2(acc2[2], acc2[3])));
    return s01.x + s01.y;
}

SLA_DEV void mma_f8_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc_, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc_), "r"(accumulate)
        : "memory");
}

SLA_DEV void mma_i8_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc_, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc_), "r"(accumulate)
        : "memory");
}

// descriptor + byte offset (the start-address field is the low 14 bits, in 16 B units)
SLA_DEV uint64_t dadd(uint64_t desc, uint32_t bytes) { return desc + (uint64_t)(bytes >> 4); }

// MODE 0: bf16 Q.K^T, fp16 P.V; 1: INT8 Q.K^T (int32 logits); 2: FP8 e4m3 Q.K^T (fp32
// logits); P.V in bf16 for both quantised modes.
template <int MODE>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
            const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_qr,
            const uint16_t *__restrict__ qraw,
            const int8_t *__restrict__ q8, const float *__restrict__ qscale, const float *__restrict__ kscale,
            const int32_t *__restrict__ idx, const float *__restrict__ hq, int N, int blk_q, int n_qb, int n_kb,
            int k_sel, int phi, uint16_t *__restrict__ out, int *status)
{
    constexpr bool QUANT = MODE != 0, INT_S = MODE == 1;
    using Cfg = AttnCfg<QUANT>;
    constexpr int NS = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    AttnSmem<QUANT> &sm =
        *reinterpret_cast<AttnSmem<QUANT> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int I = blockIdx.x, bh = blockIdx.y;
    const int32_t *sel = idx + ((size_t)bh * n_qb + I) * k_sel;
    const int n_tiles = (k_sel + 1) >> 1;
    auto n_blk = [&](int g) { return (k_sel + 1 - g) >> 1; };  // blocks of softmax group g
    volatile int *abort_flag = &sm.abort_flag;
    if (tid == 0) sm.abort_flag = global_failed(status) ? 1 : 0;
    __syncthreads();
    if (sm.abort_flag) return;  // another CTA already failed: CTA-uniform early exit

    if (tid == 0) {
        mbar_init(&sm.bar_q, 256);
        mbar_init(&sm.bar_h, 1);
        mbar_init(&sm.bar_qr, 1);
        mbar_init(&sm.bar_phiq, 256);
        mbar_init(&sm.bar_lin, 1);
        for (int d = 0; d < 3; ++d) mbar_init(&sm.drain[d], 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 2);  // one commit from each P.V issuer per tile
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.bar_s[b], 1);
            mbar_init(&sm.bar_sfree[b], 128);
            mbar_init(&sm.bar_p[b], 128);
            mbar_init(&sm.bar_pv[b], 1);
            for (int q = 0; q < 4; ++q) mbar_init(&sm.tok[b][q], 1);
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
    const uint32_t t_s = tmem, t_p = tmem + 128, t_q = tmem + 192, t_o = tmem + 256, t_l = tmem;
    uint8_t *h_s = sm.region;                       // end: 4 x [128 dims x 32 fp32]
    uint8_t *phiq_s = sm.region + 4 * kQRowsBox;    // end: 4 x [128 rows x 32 fp32]
    uint8_t *qraw_s = sm.region + 8 * kQRowsBox;    // end: 2 x [128 rows x 64 bf16] (raw Q for phi)

    // Issuing warps (producer, linear branch, Q.K^T + P.V of each group) run their
    // loops with all 32 lanes, so that stage offsets and descriptors are
    // warp-uniform, and elect one lane for each TMA / tcgen05 instruction.
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (elect_one()) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_h);
            tma_prefetch_desc(&tm_qr);
            // the linear epilogue's operands (H_I, raw Q rows) into L2 now, so that their loads
            // at the end of the CTA do not wait on HBM
            for (int c = 0; c < 4; ++c) tma_prefetch_l2_3d(&tm_h, 32 * c, 0, bh * n_qb + I);
            for (int c = 0; c < 2; ++c) tma_prefetch_l2_3d(&tm_qr, 64 * c, I * blk_q, bh);
        }
        int issued = 0;
        bool ok = true;
        for (int t = 0; ok && t < n_tiles; ++t) {
            const int s = t % NS, u = t / NS;
            if (u > 0 && !(ok = mbar_wait_warp(&sm.empty[s], (u - 1) & 1, status, abort_flag))) break;
            const int nb = min(2, k_sel - 2 * t);
            uint8_t *st = sm.region + s * Cfg::kStageBytes;
            const int J0 = __ldg(sel + 2 * t), J1 = nb > 1 ? __ldg(sel + 2 * t + 1) : 0;
            if (elect_one()) {
                mbar_expect_tx(&sm.full[s], (uint32_t)nb * Cfg::kStageBytes / 2);
                for (int x = 0; x < nb; ++x) {
                    const int J = x ? J1 : J0;
                    // K: rows 64x..64x+63 of the pair (one 128-channel int8 box, or two 64-channel bf16 boxes)
                    tma_load_3d(st + x * kBox, &tm_k, &sm.full[s], 0, J * 64, bh);
                    if (!QUANT) tma_load_3d(st + 2 * kBox + x * kBox, &tm_k, &sm.full[s], 64, J * 64, bh);
                    // V: dims 0-63 then dims 64-127, each [128 keys x 128 B] for the pair
                    tma_load_3d(st + Cfg::kKBytes + x * kBox, &tm_v, &sm.full[s], 0, J * 64, bh);
                    tma_load_3d(st + Cfg::kKBytes + 2 * kBox + x * kBox, &tm_v, &sm.full[s], 64, J * 64, bh);
                }
            }
            __syncwarp();
            issued = t + 1;
        }
        // H_I and the raw Q rows into the region once every stage is retired
        for (int s = 0; ok && s < NS; ++s) {
            int tl = -1;
            for (int t = s; t < n_tiles; t += NS) tl = t;
            if (tl >= 0) ok = mbar_wait_warp(&sm.empty[s], (tl / NS) & 1, status, abort_flag);
        }
        if (ok && elect_one()) {
            mbar_expect_tx(&sm.bar_h, 4 * kQRowsBox);
            for (int c = 0; c < 4; ++c) tma_load_3d(h_s + c * kQRowsBox, &tm_h, &sm.bar_h, 32 * c, 0, bh * n_qb + I);
            mbar_expect_tx(&sm.bar_qr, 2 * kQRowsBox);
            for (int c = 0; c < 2; ++c)
                tma_load_3d(qraw_s + c * kQRowsBox, &tm_qr, &sm.bar_qr, 64 * c, I * blk_q, bh);
        }
        __syncwarp();
        if (!ok) {  // failure: let loads in flight land before shared memory is released
            for (int s = 0; s < NS; ++s) {
                int tl = -1;
                for (int t = s; t < issued; t += NS) tl = t;
                if (tl >= 0) mbar_wait_quiet(&sm.full[s], (tl / NS) & 1, status);
            }
        } else {
            mbar_wait_quiet(&sm.bar_h, 0, status);
            mbar_wait_quiet(&sm.bar_qr, 0, status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ linear-branch MMA
        // L = phi(Q_I) H_I (tf32) into the S columns, after the softmax groups are done
        bool ok = mbar_wait_warp(&sm.bar_h, 0, status, abort_flag);
        if (ok) ok = mbar_wait_warp(&sm.bar_phiq, 0, status, abort_flag);
        if (ok) {
            tc_fence_after();
            constexpr uint32_t id_lin = idesc(1, 2, 2, 0, 0, 128, 128);  // f32 <- tf32 x tf32, K-major
            const uint64_t pd = sdesc_sw128(smem_u32(phiq_s), 16, 1024), hd = sdesc_sw128(smem_u32(h_s), 16, 1024);
            if (elect_one()) {
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const uint32_t off = (k >> 2) * kQRowsBox + (k & 3) * 32;
                    mma_tf32(t_l, dadd(pd, off), dadd(hd, off), id_lin, k > 0 ? 1u : 0u);
                }
                mma_commit(&sm.bar_lin);
            }
            __syncwarp();
        }
        if (elect_one()) {
            mma_commit(&sm.drain[0]);
            mbar_wait_quiet(&sm.drain[0], 0, status);  // this thread's MMAs retired before TMEM is released
        }
        __syncwarp();
    } else if (warp >= 10) {
        // ------------------------------------------------------------ Q.K^T + P.V issuer of group g
        const int g = warp - 10;
        // S32 <- s8 x s8 (INT8), F32 <- e4m3 x e4m3 (FP8), F32 <- bf16 x bf16
        constexpr uint32_t id_qk = MODE == 1   ? idesc(2, 1, 1, 0, 0, 128, 64)
                                   : MODE == 2 ? idesc(1, 0, 0, 0, 0, 128, 64)
                                               : idesc(1, 1, 1, 0, 0, 128, 64);
        constexpr uint32_t id_pv = QUANT ? idesc(1, 1, 1, 0, 1, 128, 128) : idesc(1, 0, 0, 0, 1, 128, 128);
        const uint64_t kd0 = sdesc_sw128(smem_u32(sm.region), 16, 1024);
        const uint64_t vd0 = sdesc_sw128(smem_u32(sm.region + Cfg::kKBytes), 2 * kBox, 1024);
        const uint32_t s_g = t_s + 64 * g, o_g = t_o + 128 * g, p_g = t_p + 32 * g;
        const int nb = n_blk(g);
        bool ok = true;
        // S_g = Q K_j^T for this group's block of tile t (K rows of block g of the pair)
        auto issue_qk = [&](int t) {
            if (!(ok = mbar_wait_warp(&sm.full[t % NS], (t / NS) & 1, status, abort_flag))) return;
            if (t > 0 && !(ok = mbar_wait_warp(&sm.bar_sfree[g], (t - 1) & 1, status, abort_flag))) return;
            tc_fence_after();
            const uint64_t kd = dadd(kd0, (t % NS) * Cfg::kStageBytes + g * kBox);
            if (elect_one()) {
                if (MODE == 1) {  // K-step of 32 int8 = 8 TMEM columns of Q
#pragma unroll
                    for (int k = 0; k < 4; ++k) mma_i8_tmem_a(s_g, t_q + 8 * k, kd + 2 * k, id_qk, k > 0 ? 1u : 0u);
                } else if (MODE == 2) {  // K-step of 32 e4m3 = 8 TMEM columns of Q
#pragma unroll
                    for (int k = 0; k < 4; ++k) mma_f8_tmem_a(s_g, t_q + 8 * k, kd + 2 * k, id_qk, k > 0 ? 1u : 0u);
                } else {  // K-step of 16 bf16 = 8 TMEM columns of Q
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_f16_tmem_a(s_g, t_q + 8 * k, kd + (k >> 2) * (2 * kBox >> 4) + 2 * (k & 3), id_qk,
                                       k > 0 ? 1u : 0u);
                }
                mma_commit(&sm.bar_s[g]);
            }
            __syncwarp();
        };
        if (nb > 0) {
            ok = mbar_wait_warp(&sm.bar_q, 0, status, abort_flag);
            if (ok) issue_qk(0);
        }
        for (int t = 0; ok && t < n_tiles; ++t) {
            if (t < nb) {
                if (t + 1 < nb) {  // next logits as soon as this group has read S
                    issue_qk(t + 1);
                    if (!ok) break;
                }
                if (!(ok = mbar_wait_warp(&sm.bar_p[g], t & 1, status, abort_flag))) break;
                tc_fence_after();
                const uint64_t vd = dadd(vd0, (t % NS) * Cfg::kStageBytes + g * kBox);  // this block's rows
                if (elect_one()) {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_f16_tmem_a(o_g, p_g + 8 * k, vd + 128 * k, id_pv, (t > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&sm.bar_pv[g]);
                }
                __syncwarp();
            }
            if (elect_one()) mma_commit(&sm.empty[t % NS]);  // stage t free once both groups' MMAs retired
            __syncwarp();
        }
        if (elect_one()) {
            mma_commit(&sm.drain[1 + g]);
            mbar_wait_quiet(&sm.drain[1 + g], 0, status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax / epilogue
        const int g = (warp - 2) >> 2;                  // group: key blocks 2t + g
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;              // query row within the tile (= TMEM lane)
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int i = I * blk_q + r;
        const bool row_valid = r < blk_q && i < N;
        // every wait below is made warp-uniform so that warp-collective tcgen05
        // loads/stores and vote instructions are always reached by all lanes
        auto wait_all = [&](uint64_t *bar, uint32_t par) {
            const bool w = mbar_wait(bar, par, status, abort_flag);
            return __all_sync(0xffffffffu, w);
        };
        if (g == 0) sm.z[r] = __ldg(hq + ((size_t)bh * n_qb + I) * kStateCols + kD * kD + r);
        // Q (INT8 codes, or bf16 without quantisation) into tensor memory: row r -> lane r, four
        // int8 (two bf16) per 32-bit column; group g writes its half of the columns
        if (k_sel > 0) {
            const bool qrow = i < N;  // rows of the next block (blk_q = 64) or past N: anything finite
            if (QUANT) {
                const uint4 *src = reinterpret_cast<const uint4 *>(q8 + ((size_t)bh * N + (qrow ? i : 0)) * kD) + 4 * g;
                uint32_t w[16];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint4 x = qrow ? __ldg(src + u) : make_uint4(0, 0, 0, 0);
                    w[4 * u] = x.x; w[4 * u + 1] = x.y; w[4 * u + 2] = x.z; w[4 * u + 3] = x.w;
                }
                tmem_st16(t_q + lane_off + 16 * g, w);
            } else {
                const uint4 *src = reinterpret_cast<const uint4 *>(qraw + ((size_t)bh * N + (qrow ? i : 0)) * kD) + 8 * g;
                uint32_t w[32];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint4 x = qrow ? __ldg(src + u) : make_uint4(0, 0, 0, 0);
                    w[4 * u] = x.x; w[4 * u + 1] = x.y; w[4 * u + 2] = x.z; w[4 * u + 3] = x.w;
                }
                tmem_st32(t_q + lane_off + 32 * g, w);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(&sm.bar_q);
        if (g == 1) {  // group 0 takes the first exponential phase
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.tok[0][quarter]);
        }

        // ---- sparse loop: this group's key blocks j = 2t + g
        const float sq = QUANT ? __ldg(qscale + (size_t)bh * n_qb + I) : 0.0f;
        const float kscale_log2 = kLog2e * kInvSqrtD;
        constexpr float kBias = 12582912.0f;  // 1.5 * 2^23: int32 d + bias bits read as float 12582912 + d
        const uint32_t s_own = t_s + 64 * g + lane_off, p_own = t_p + 32 * g + lane_off;
        const uint32_t o_own = t_o + 128 * g + lane_off;
        // per-tile block index and key scale, prefetched ahead of use
        auto blk_of = [&](int t) { return (2 * t + g < k_sel) ? __ldg(sel + 2 * t + g) : -1; };
        int J_a = blk_of(0), J_b = blk_of(1);
        float ks_a = (QUANT && J_a >= 0) ? __ldg(kscale + (size_t)bh * n_kb + J_a) : 0.0f;
        float m_used = -INFINITY, l = 0.0f;
        bool ok = true;
        const int nb = n_blk(g);
        // Phase tests are issued ahead of use (see mbar_test); a negative answer
        // falls back to the bounded wait.
        bool s_ready = false;
        for (int t = 0; ok && t < nb; ++t) {
            const int J = J_a;
            const float c = QUANT ? sq * ks_a * kscale_log2 : kscale_log2;
            if (t + 1 < nb) {
                J_a = J_b;
                if (QUANT) ks_a = __ldg(kscale + (size_t)bh * n_kb + J_b);
            }
            if (t + 2 < nb) J_b = blk_of(t + 2);
            if (!__all_sync(0xffffffffu, s_ready) && !(ok = wait_all(&sm.bar_s[g], t & 1))) break;
            tc_fence_after();
            uint32_t sv[64];
            tmem_ld32(s_own, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
            tmem_ld32(s_own + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.bar_sfree[g]);  // S_g may be rewritten now
            const bool tok_ready = mbar_test(&sm.tok[g][quarter], t & 1);
            const int valid = min(64, N - J * 64);
            // the two paths are separate instantiations so the full-tile path carries no masking
            const float tmax = valid == 64 ? tile_max<INT_S, false>(sv, 64, c) : tile_max<INT_S, true>(sv, valid, c);
            const float m_new = fmaxf(m_used, tmax);
            const bool need = m_new > m_used + kRescaleThreshold;  // also true on the first block
            float alpha = 1.0f;
            if (need) {
                alpha = ex2(m_used - m_new);  // 0 when m_used = -inf
                m_used = m_new;
                l *= alpha;
            }
            // exponential phase, alternating with the other group's warp on this sub-partition
            if (!__all_sync(0xffffffffu, tok_ready) && !(ok = wait_all(&sm.tok[g][quarter], t & 1))) break;
            const bool pv_ready = t == 0 || mbar_test(&sm.bar_pv[g], (t - 1) & 1);
            uint32_t pk[32];
            const float off = INT_S ? -fmaf(kBias, c, m_used) : -m_used;
            if (valid == 64) l += tile_exp<QUANT, false>(sv, 64, c, off, pk);
            else l += tile_exp<QUANT, true>(sv, valid, c, off, pk);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.tok[g ^ 1][quarter]);
            // P and O of this group are free/stable once its previous P.V has retired
            if (!__all_sync(0xffffffffu, pv_ready) && !(ok = wait_all(&sm.bar_pv[g], (t - 1) & 1))) break;
            if (t > 0 && __any_sync(0xffffffffu, need)) {  // rescale O of this group
                tc_fence_after();
                uint32_t o[32];
#pragma unroll 1
                for (int c0 = 0; c0 < kD; c0 += 32) {
                    tmem_ld32(o_own + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(o_own + c0, o);
                }
            }
            tmem_st32(p_own, pk);  // P packed to bf16 (fp16 without quantisation)
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&sm.bar_p[g]);
            if (t + 1 < nb) s_ready = mbar_test(&sm.bar_s[g], (t + 1) & 1);
        }
        // ---- linear branch operands: wait for every P.V (the ring is then free), then phi(Q) + den
        if (ok && n_blk(0) > 0) ok = wait_all(&sm.bar_pv[0], (n_blk(0) - 1) & 1);
        if (ok && n_blk(1) > 0) ok = wait_all(&sm.bar_pv[1], (n_blk(1) - 1) & 1);
        named_bar_sync(5, 256);  // every group past its P.V waits (z is also visible now)
        float den = 0.0f;
        if (ok) ok = wait_all(&sm.bar_qr, 0);  // raw Q rows of this tile (rows past N read as 0)
        if (ok) {
#pragma unroll 2
            for (int uu = 0; uu < 8; ++uu) {  // group g: channels 64g..64g+63, 8 per iteration
                const int u = 8 * g + uu;
                const uint4 w = *reinterpret_cast<const uint4 *>(qraw_s + g * kQRowsBox + sw128_off(r, uu));
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                float f[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    f[2 * e] = row_valid ? phi_tf32(__uint_as_float(ww[e] << 16), phi) : 0.0f;
                    f[2 * e + 1] = row_valid ? phi_tf32(__uint_as_float(ww[e] & 0xFFFF0000u), phi) : 0.0f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) den = fmaf(f[e], sm.z[8 * u + e], den);
                // channels 8u..8u+7 = chunk (u/4), 16-byte units (2u)%8 and (2u+1)%8 of row r
                uint8_t *base = phiq_s + (u >> 2) * kQRowsBox;
                *reinterpret_cast<float4 *>(base + sw128_off(r, (2 * u) & 7)) = make_float4(f[0], f[1], f[2], f[3]);
                *reinterpret_cast<float4 *>(base + sw128_off(r, (2 * u + 1) & 7)) = make_float4(f[4], f[5], f[6], f[7]);
            }
            fence_async_smem();
        }
        mbar_arrive(&sm.bar_phiq);
        // ---- epilogue: merge the two groups' partial softmax; group g writes output columns 64g..64g+63
        sm.fin[g][0][r] = m_used;
        sm.fin[g][1][r] = l;
        sm.fin[g][2][r] = den;
        named_bar_sync(5, 256);
        if (ok) ok = wait_all(&sm.bar_lin, 0);
        if (ok) {
            tc_fence_after();
            const int n0 = n_blk(0), n1 = n_blk(1);
            const float m0 = sm.fin[0][0][r], l0 = sm.fin[0][1][r], m1 = sm.fin[1][0][r], l1 = sm.fin[1][1][r];
            const float m = fmaxf(m0, m1);
            const float s0 = n0 > 0 ? ex2(m0 - m) : 0.0f, s1 = n1 > 0 ? ex2(m1 - m) : 0.0f;
            const float lt = l0 * s0 + l1 * s1;
            const float inv_l = lt > 0.0f ? 1.0f / lt : 0.0f;
            const float w0 = s0 * inv_l, w1 = s1 * inv_l;
            const float dt = sm.fin[0][2][r] + sm.fin[1][2][r];
            const float inv_den = dt != 0.0f ? 1.0f / dt : 0.0f;
            uint16_t *orow = out + ((size_t)bh * N + (row_valid ? i : 0)) * kD + 64 * g;
            const uint32_t o0 = t_o + lane_off + 64 * g, o1 = t_o + 128 + lane_off + 64 * g;
#pragma unroll 1
            for (int c0 = 0; c0 < 64; c0 += 32) {
                uint32_t lr[32], a0[32], a1[32];
                tmem_ld32(t_l + lane_off + 64 * g + c0, lr);
                if (n0 > 0) tmem_ld32(o0 + c0, a0);
                if (n1 > 0) tmem_ld32(o1 + c0, a1);
                tmem_wait_ld();
                uint32_t pkk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float v[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float x = __uint_as_float(lr[2 * e + h]) * inv_den;
                        if (n0 > 0) x = fmaf(__uint_as_float(a0[2 * e + h]), w0, x);
                        if (n1 > 0) x = fmaf(__uint_as_float(a1[2 * e + h]), w1, x);
                        v[h] = x;
                    }
                    pkk[e] = pack_bf16x2(v[0], v[1]);
                }
                if (row_valid) {
                    uint4 *o4 = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        o4[e] = make_uint4(pkk[4 * e], pkk[4 * e + 1], pkk[4 * e + 2], pkk[4 * e + 3]);
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

template <int MODE>
cudaError_t launch_attn_t(const void *q, const void *k, const void *v, const int8_t *q8, const int8_t *k8,
                          const float *qscale, const float *kscale, const int32_t *idx, const float *hq,
                          const Geometry &g, int phi, void *out, int *status, cudaStream_t s)
{
    constexpr bool QUANT = MODE != 0;
    CUtensorMap tk, tv, th, tq;
    const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)g.N, (uint64_t)g.BH};
    if (QUANT) {
        const uint64_t st[2] = {(uint64_t)kD, (uint64_t)g.N * kD};
        const uint32_t bk[3] = {128, 64, 1};
        if (!encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, k8, dims, st, bk)) return cudaErrorInvalidValue;
    } else {
        const uint64_t st[2] = {(uint64_t)kD * 2, (uint64_t)g.N * kD * 2};
        const uint32_t bk[3] = {64, 64, 1};
        if (!encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dims, st, bk)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t st[2] = {(uint64_t)kD * 2, (uint64_t)g.N * kD * 2};
        const uint32_t bv[3] = {64, 64, 1};
        const CUtensorMapDataType vt = QUANT ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        if (!encode_tmap(&tv, vt, 3, v, dims, st, bv)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t hd[3] = {(uint64_t)kD, (uint64_t)kD, (uint64_t)g.BH * g.n_qb};
        const uint64_t st[2] = {(uint64_t)kD * 4, (uint64_t)kStateCols * 4};
        const uint32_t bh[3] = {32, 128, 1};
        if (!encode_tmap(&th, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, hq, hd, st, bh)) return cudaErrorInvalidValue;
    }
    {
        // raw Q rows of a query block for phi(Q): [BH, N, 128] bf16, boxes of 64 channels x 128 rows
        const uint64_t st[2] = {(uint64_t)kD * 2, (uint64_t)g.N * kD * 2};
        const uint32_t bq[3] = {64, 128, 1};
        if (!encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, dims, st, bq)) return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(AttnSmem<QUANT>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(g.n_qb, g.BH);
    attn_kernel<MODE><<<grid, kAttnThreads, smem, s>>>(tk, tv, th, tq, static_cast<const uint16_t *>(q), q8, qscale,
                                                        kscale, idx, hq, g.N, g.blk_q, g.n_qb, g.n_kb, g.k_sel, phi,
                                                        static_cast<uint16_t *>(out), status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const void *q, const void *k, const void *v, const int8_t *q8, const int8_t *k8,
                             const float *qscale, const float *kscale, const int32_t *idx, const float *hq,
                             const Geometry &g, int phi, void *out, int *status, cudaStream_t s)
{
    if (g.quant == 2) return launch_attn_t<2>(q, k, v, q8, k8, qscale, kscale, idx, hq, g, phi, out, status, s);
    if (g.quant == 1) return launch_attn_t<1>(q, k, v, q8, k8, qscale, kscale, idx, hq, g, phi, out, status, s);
    return launch_attn_t<0>(q, k, v, q8, k8, qscale, kscale, idx, hq, g, phi, out, status, s);
}

cudaError_t set_wait_budget_attention(long long cycles) { return set_tu_wait_budget(cycles); }

}  // namespace sla
