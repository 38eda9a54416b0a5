// sla_attention.cu -- fused block-sparse attention + linear epilogue of the
// SageSLA forward: one CTA per (batch*head, query block), two CTAs per SM.
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
// Linear branch ("TurboDiffusion技术架构解析" §2.1, linear attention
// phi(Q)(phi(K)^T V)): after the sparse loop the row's normaliser phi(q) . Z_I
// is computed on the CUDA cores, and A = phi(q) * l / (phi(q) . Z_I) (l: the
// row's softmax sum) is written to tensor memory in tf32, so that one tf32 MMA
// O += A H_I leaves O / l = O_sparse + O_linear in the same accumulator.
//
// Tiling.  One softmax warpgroup takes the query block's selected key blocks
// in selection order, one M=128, N=64 Q.K^T per block, with its S, P, O and
// running (max, sum) in tensor memory and registers.  Two such CTAs share an
// SM (256 TMEM columns and ~99 KB of shared memory each), so one CTA's
// prologue (Q codes, first K/V tiles) and epilogue (linear branch, output
// store) overlap the other CTA's main loop, and their exponential phases
// interleave on the MUFU units.
//
// Issue.  tcgen05 and mbarrier operations cost tens of cycles each on the
// issuing thread, so a dedicated warp issues the Q.K^T and P.V MMAs.
// Dependencies go through mbarriers only: S is rewritten once it has been
// read; P is rewritten once the previous P.V has completed.
//
// Shared-memory bandwidth (128 B/clk, shared by TMA writes and tensor-core
// operand reads): the A operands of the quantised modes live in tensor memory
// -- Q (written once per CTA from registers) and P (two 16-bit values per
// 32-bit column) -- so per key block only K and V cross shared memory, through
// a ring of four stages (two without quantisation, whose bf16 Q tile stays in
// shared memory as the Q.K^T A operand).  The linear branch runs at the end,
// reusing the ring for H_I and the raw Q rows.
//
// Roles (192 threads): warp 0 TMA producer, warp 1 MMA issuer and TMEM owner,
// warps 2-5 softmax and epilogue (one query row per thread, one TMEM lane
// quarter per warp).  TMEM columns: S at 0, P at 64, Q codes at 96, O at 128;
// the linear branch's A operand takes columns 0-127 at the end.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "sla_internal.h"
#include "sla_ptx.cuh"

namespace sla {
namespace {

constexpr int kAttnThreads = 192;
constexpr uint32_t kAttnTmemCols = 256;
constexpr uint32_t kBox = 64 * 128;          // [64 rows x 128 B]
constexpr uint32_t kQRowsBox = 128 * 128;    // [128 rows x 128 B]
constexpr uint32_t kRegion = 6 * kQRowsBox;  // 96 KB: the K/V ring, then H_I (64 KB) + raw Q rows (32 KB)
constexpr uint32_t kQRawOff = 4 * kQRowsBox; // raw Q rows (and the bf16 Q tile without quantisation)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;    // log2 units: P may grow to 2^8 before O is rescaled
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1 / sqrt(128)

template <bool QUANT>  // QUANT: 8-bit Q/K codes (INT8 or FP8)
struct AttnCfg {
    static constexpr uint32_t kKBytes = QUANT ? kBox : 2 * kBox;  // K of one key block (int8, or two bf16 boxes)
    static constexpr uint32_t kVBytes = 2 * kBox;                 // V of one key block: dims 0-63, 64-127
    static constexpr uint32_t kStageBytes = kKBytes + kVBytes;
    static constexpr int kStages = QUANT ? 4 : 2;
    // quantised: the ring fills the region; otherwise it ends where the bf16 Q tile begins
    static_assert(kStages * kStageBytes <= (QUANT ? kRegion : kQRawOff), "ring fits");
};

struct AttnSmem {
    alignas(1024) uint8_t region[kRegion];
    float z[kD];
    uint64_t full[4], empty[4];
    uint64_t bar_q, bar_s, bar_sfree, bar_p, bar_pv, bar_h, bar_qr, bar_phiq, bar_lin, drain;
    uint32_t tmem_base;
    int abort_flag;
};

SLA_DEV float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
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

// tf32 MMA with A in tensor memory (rows = lanes, one 32-bit K element per column)
SLA_DEV void mma_tf32_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc_, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc_), "r"(accumulate)
        : "memory");
}

// phi of the 8 bf16 channels of one 16-byte unit of a raw Q row (fp32, not rounded)
SLA_DEV void phi8(const uint4 &w, int phi, float (&f)[8])
{
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float lo = __uint_as_float(ww[e] << 16), hi = __uint_as_float(ww[e] & 0xFFFF0000u);
        const float elo = ex2(fminf(lo, 0.0f) * kLog2e), ehi = ex2(fminf(hi, 0.0f) * kLog2e);
        f[2 * e] = phi == 1 ? fmaxf(lo, 0.0f) : (lo > 0.0f ? lo + 1.0f : elo);
        f[2 * e + 1] = phi == 1 ? fmaxf(hi, 0.0f) : (hi > 0.0f ? hi + 1.0f : ehi);
    }
}

// MODE 0: bf16 Q.K^T, fp16 P.V; 1: INT8 Q.K^T (int32 logits); 2: FP8 e4m3 Q.K^T (fp32
// logits); P.V in bf16 for both quantised modes.
template <int MODE>
__global__ void __launch_bounds__(kAttnThreads, 2)
attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
            const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_qr,
            const int8_t *__restrict__ q8, const float *__restrict__ qscale, const float *__restrict__ kscale,
            const int32_t *__restrict__ idx, const float *__restrict__ hq, int N, int blk_q, int n_qb, int n_kb,
            int k_sel, int phi, uint16_t *__restrict__ out, int *status)
{
    constexpr bool QUANT = MODE != 0, INT_S = MODE == 1;
    using Cfg = AttnCfg<QUANT>;
    constexpr int NS = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    AttnSmem &sm = *reinterpret_cast<AttnSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int I = blockIdx.x, bh = blockIdx.y;
    const int32_t *sel = idx + ((size_t)bh * n_qb + I) * k_sel;
    volatile int *abort_flag = &sm.abort_flag;
    if (tid == 0) sm.abort_flag = global_failed(status) ? 1 : 0;
    __syncthreads();
    if (sm.abort_flag) return;  // another CTA already failed: CTA-uniform early exit

    if (tid == 0) {
        mbar_init(&sm.bar_q, QUANT ? 128 : 1);  // codes stored by the 128 softmax threads / the Q tile's TMA
        mbar_init(&sm.bar_s, 1);
        mbar_init(&sm.bar_sfree, 128);
        mbar_init(&sm.bar_p, 128);
        mbar_init(&sm.bar_pv, 1);
        mbar_init(&sm.bar_h, 1);
        mbar_init(&sm.bar_qr, 1);
        mbar_init(&sm.bar_phiq, 128);
        mbar_init(&sm.bar_lin, 1);
        mbar_init(&sm.drain, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, kAttnTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // S at 0 (64 columns), P at 64 (32), Q codes at 96 (32), O at 128 (128); at the end the
    // linear branch's A operand (128 tf32 columns) replaces S, P and Q
    const uint32_t t_s = tmem, t_p = tmem + 64, t_q = tmem + 96, t_a = tmem, t_o = tmem + 128;
    uint8_t *h_s = sm.region;                       // end: H_I, 4 x [128 dims x 32 fp32]
    uint8_t *qraw_s = sm.region + kQRawOff;         // raw Q rows, 2 x [128 rows x 64 bf16]

    // Issuing warps (producer, MMA issuer) run their loops with all 32 lanes, so that stage
    // offsets and descriptors are warp-uniform, and elect one lane for each TMA / tcgen05 instruction.
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (elect_one()) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_h);
            tma_prefetch_desc(&tm_qr);
            // the linear epilogue's operands into L2 now, so that their loads at the end do not wait on HBM
            tma_prefetch_l2_4d(&tm_h, 0, 0, 0, bh * n_qb + I);
            if (QUANT) {
                tma_prefetch_l2_4d(&tm_qr, 0, I * blk_q, 0, bh);
            } else {  // the bf16 Q tile: A operand of Q.K^T, and the raw Q of phi at the end
                mbar_expect_tx(&sm.bar_q, 2 * kQRowsBox);
                tma_load_4d(qraw_s, &tm_qr, &sm.bar_q, 0, I * blk_q, 0, bh);
            }
        }
        __syncwarp();
        int issued = 0;
        bool ok = true;
        for (int t = 0; ok && t < k_sel; ++t) {
            const int s = t % NS, u = t / NS;
            if (u > 0 && !(ok = mbar_wait_warp(&sm.empty[s], (u - 1) & 1, status, abort_flag))) break;
            uint8_t *st = sm.region + s * Cfg::kStageBytes;
            const int J = __ldg(sel + t);
            if (elect_one()) {
                mbar_expect_tx(&sm.full[s], Cfg::kStageBytes);
                // K: one 128-channel int8 box, or the two 64-channel halves of the bf16 rows; V: the two
                // halves of its rows (dims 0-63, then 64-127).  One copy each: a copy costs the issuing
                // CTA about the same whatever its size
                if (QUANT) tma_load_3d(st, &tm_k, &sm.full[s], 0, J * 64, bh);
                else tma_load_4d(st, &tm_k, &sm.full[s], 0, J * 64, 0, bh);
                tma_load_4d(st + Cfg::kKBytes, &tm_v, &sm.full[s], 0, J * 64, 0, bh);
            }
            __syncwarp();
            issued = t + 1;
        }
        // H_I (and, quantised, the raw Q rows) into the ring once every stage is retired
        for (int s = 0; ok && s < NS; ++s) {
            int tl = -1;
            for (int t = s; t < k_sel; t += NS) tl = t;
            if (tl >= 0) ok = mbar_wait_warp(&sm.empty[s], (tl / NS) & 1, status, abort_flag);
        }
        if (ok && elect_one()) {
            mbar_expect_tx(&sm.bar_h, 4 * kQRowsBox);
            tma_load_4d(h_s, &tm_h, &sm.bar_h, 0, 0, 0, bh * n_qb + I);
            if (QUANT) {
                mbar_expect_tx(&sm.bar_qr, 2 * kQRowsBox);
                tma_load_4d(qraw_s, &tm_qr, &sm.bar_qr, 0, I * blk_q, 0, bh);
            }
        }
        __syncwarp();
        // before shared memory is released: every load issued has landed
        if (!ok) {
            for (int s = 0; s < NS; ++s) {
                int tl = -1;
                for (int t = s; t < issued; t += NS) tl = t;
                if (tl >= 0) mbar_wait_quiet(&sm.full[s], (tl / NS) & 1, status);
            }
        } else {
            mbar_wait_quiet(&sm.bar_h, 0, status);
            if (QUANT) mbar_wait_quiet(&sm.bar_qr, 0, status);
        }
        if (!QUANT) mbar_wait_quiet(&sm.bar_q, 0, status);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // S32 <- s8 x s8 (INT8), F32 <- e4m3 x e4m3 (FP8), F32 <- bf16 x bf16
        constexpr uint32_t id_qk = MODE == 1   ? idesc(2, 1, 1, 0, 0, 128, 64)
                                   : MODE == 2 ? idesc(1, 0, 0, 0, 0, 128, 64)
                                               : idesc(1, 1, 1, 0, 0, 128, 64);
        constexpr uint32_t id_pv = QUANT ? idesc(1, 1, 1, 0, 1, 128, 128) : idesc(1, 0, 0, 0, 1, 128, 128);
        constexpr uint32_t id_lin = idesc(1, 2, 2, 0, 0, 128, 128);  // f32 <- tf32 x tf32, K-major
        const uint64_t kd0 = sdesc_sw128(smem_u32(sm.region), 16, 1024);
        const uint64_t vd0 = sdesc_sw128(smem_u32(sm.region + Cfg::kKBytes), kBox, 1024);
        const uint64_t qd0 = sdesc_sw128(smem_u32(qraw_s), 16, 1024);  // the bf16 Q tile (quantisation off)
        bool ok = true;
        // S = Q K_J^T for key block t of the selection
        auto issue_qk = [&](int t) {
            if (!(ok = mbar_wait_warp(&sm.full[t % NS], (t / NS) & 1, status, abort_flag))) return;
            if (t > 0 && !(ok = mbar_wait_warp(&sm.bar_sfree, (t - 1) & 1, status, abort_flag))) return;
            tc_fence_after();
            const uint64_t kd = dadd(kd0, (t % NS) * Cfg::kStageBytes);
            if (elect_one()) {
                if (MODE == 1) {  // K-step of 32 int8 = 8 TMEM columns of Q
#pragma unroll
                    for (int k = 0; k < 4; ++k) mma_i8_tmem_a(t_s, t_q + 8 * k, dadd(kd, 32 * k), id_qk, k > 0 ? 1u : 0u);
                } else if (MODE == 2) {  // K-step of 32 e4m3 = 8 TMEM columns of Q
#pragma unroll
                    for (int k = 0; k < 4; ++k) mma_f8_tmem_a(t_s, t_q + 8 * k, dadd(kd, 32 * k), id_qk, k > 0 ? 1u : 0u);
                } else {  // K-step of 16 bf16: 32 bytes of a 64-channel box
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t off = (k >> 2) * kQRowsBox + (k & 3) * 32, koff = (k >> 2) * kBox + (k & 3) * 32;
                        mma_bf16(t_s, dadd(qd0, off), dadd(kd, koff), id_qk, k > 0 ? 1u : 0u);
                    }
                }
                mma_commit(&sm.bar_s);
            }
            __syncwarp();
        };
        if (k_sel > 0) {
            ok = mbar_wait_warp(&sm.bar_q, 0, status, abort_flag);
            if (ok) issue_qk(0);
        }
        for (int t = 0; ok && t < k_sel; ++t) {
            if (t + 1 < k_sel) {  // next logits as soon as S has been read
                issue_qk(t + 1);
                if (!ok) break;
            }
            if (!(ok = mbar_wait_warp(&sm.bar_p, t & 1, status, abort_flag))) break;
            tc_fence_after();
            const uint64_t vd = dadd(vd0, (t % NS) * Cfg::kStageBytes);
            if (elect_one()) {
#pragma unroll
                for (int k = 0; k < 4; ++k)  // K-step of 16 keys = 8 TMEM columns of P, 2 KB of V rows
                    mma_f16_tmem_a(t_o, t_p + 8 * k, dadd(vd, 2048 * k), id_pv, (t > 0 || k > 0) ? 1u : 0u);
                mma_commit(&sm.bar_pv);
                mma_commit(&sm.empty[t % NS]);  // the stage is free once Q.K^T and P.V of block t retired
            }
            __syncwarp();
        }
        // linear branch: O += A H_I, A = phi(Q) scaled per row (tf32, TMEM columns 0-127)
        if (ok) ok = mbar_wait_warp(&sm.bar_h, 0, status, abort_flag);
        if (ok) ok = mbar_wait_warp(&sm.bar_phiq, 0, status, abort_flag);
        if (ok) {
            tc_fence_after();
            const uint64_t hd = sdesc_sw128(smem_u32(h_s), 16, 1024);
            if (elect_one()) {
#pragma unroll
                for (int k = 0; k < 16; ++k)  // K-step of 8 tf32 channels: 32 bytes of a 32-channel box
                    mma_tf32_tmem_a(t_o, t_a + 8 * k, dadd(hd, (k >> 2) * kQRowsBox + (k & 3) * 32), id_lin,
                                    (k > 0 || k_sel > 0) ? 1u : 0u);
                mma_commit(&sm.bar_lin);
            }
            __syncwarp();
        }
        if (elect_one()) {
            mma_commit(&sm.drain);
            mbar_wait_quiet(&sm.drain, 0, status);  // this thread's MMAs retired before TMEM is released
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax / epilogue
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
        sm.z[r] = __ldg(hq + ((size_t)bh * n_qb + I) * kStateCols + kD * kD + r);
        if (QUANT) {
            // Q codes into tensor memory: row r -> lane r, four codes per 32-bit column
            if (k_sel > 0) {
                const bool qrow = i < N;  // rows of the next block (blk_q = 64) or past N: anything finite
                const uint4 *src = reinterpret_cast<const uint4 *>(q8 + ((size_t)bh * N + (qrow ? i : 0)) * kD);
                uint32_t w[32];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint4 x = qrow ? __ldg(src + u) : make_uint4(0, 0, 0, 0);
                    w[4 * u] = x.x; w[4 * u + 1] = x.y; w[4 * u + 2] = x.z; w[4 * u + 3] = x.w;
                }
                tmem_st32(t_q + lane_off, w);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(&sm.bar_q);
        }
        named_bar_sync(1, 128);  // z is visible to every softmax thread

        // ---- sparse loop over the selected key blocks, in selection order
        const float sq = QUANT ? __ldg(qscale + (size_t)bh * n_qb + I) : 0.0f;
        const float kscale_log2 = kLog2e * kInvSqrtD;
        constexpr float kBias = 12582912.0f;  // 1.5 * 2^23: int32 d + bias bits read as float 12582912 + d
        const uint32_t s_own = t_s + lane_off, p_own = t_p + lane_off, o_own = t_o + lane_off;
        // block index and key scale of the next blocks, prefetched ahead of use
        auto blk_of = [&](int t) { return t < k_sel ? __ldg(sel + t) : -1; };
        int J_a = blk_of(0), J_b = blk_of(1);
        float ks_a = (QUANT && J_a >= 0) ? __ldg(kscale + (size_t)bh * n_kb + J_a) : 0.0f;
        float m_used = -INFINITY, l = 0.0f;
        bool ok = true;
        // Phase tests are issued ahead of use (see mbar_test); a negative answer
        // falls back to the bounded wait.
        bool s_ready = false;
        for (int t = 0; ok && t < k_sel; ++t) {
            const int J = J_a;
            const float c = QUANT ? sq * ks_a * kscale_log2 : kscale_log2;
            if (t + 1 < k_sel) {
                J_a = J_b;
                if (QUANT) ks_a = __ldg(kscale + (size_t)bh * n_kb + J_b);
            }
            if (t + 2 < k_sel) J_b = blk_of(t + 2);
            if (!__all_sync(0xffffffffu, s_ready) && !(ok = wait_all(&sm.bar_s, t & 1))) break;
            tc_fence_after();
            uint32_t sv[64];
            tmem_ld32(s_own, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
            tmem_ld32(s_own + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sm.bar_sfree);  // S may be rewritten now
            const bool pv_ready = t == 0 || mbar_test(&sm.bar_pv, (t - 1) & 1);
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
            uint32_t pk[32];
            const float off = INT_S ? -fmaf(kBias, c, m_used) : -m_used;
            if (valid == 64) l += tile_exp<QUANT, false>(sv, 64, c, off, pk);
            else l += tile_exp<QUANT, true>(sv, valid, c, off, pk);
            // P and O are free/stable once the previous P.V has retired
            if (!__all_sync(0xffffffffu, pv_ready) && !(ok = wait_all(&sm.bar_pv, (t - 1) & 1))) break;
            if (t > 0 && __any_sync(0xffffffffu, need)) {  // rescale O
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
            mbar_arrive(&sm.bar_p);
            if (t + 1 < k_sel) s_ready = mbar_test(&sm.bar_s, (t + 1) & 1);
        }

        // ---- linear branch: A = phi(q) * l / (phi(q) . Z_I) in tf32, so that the MMA O += A H_I
        // leaves O / l = O_sparse + O_linear
        if (ok && k_sel > 0) ok = wait_all(&sm.bar_pv, (k_sel - 1) & 1);  // P and S columns are free
        if (ok) ok = wait_all(QUANT ? &sm.bar_qr : &sm.bar_q, 0);         // raw Q rows (past N: zeros)
        const float l_eff = k_sel > 0 ? l : 1.0f;  // no sparse blocks: O is the linear MMA's alone
        if (ok) {
            float den = 0.0f;
#pragma unroll 2
            for (int u = 0; u < 16; ++u) {  // channels 8u..8u+7
                const uint4 w = *reinterpret_cast<const uint4 *>(qraw_s + (u >> 3) * kQRowsBox + sw128_off(r, u & 7));
                float f[8];
                phi8(w, phi, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) den = fmaf(f[e], sm.z[8 * u + e], den);
            }
            const float scale = (row_valid && den != 0.0f) ? __fdiv_rn(l_eff, den) : 0.0f;
#pragma unroll 1
            for (int c0 = 0; c0 < kD; c0 += 32) {
                uint32_t a[32];
#pragma unroll
                for (int uu = 0; uu < 4; ++uu) {
                    const int u = (c0 >> 3) + uu;
                    const uint4 w =
                        *reinterpret_cast<const uint4 *>(qraw_s + (u >> 3) * kQRowsBox + sw128_off(r, u & 7));
                    float f[8];
                    phi8(w, phi, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) a[8 * uu + e] = __float_as_uint(to_tf32(f[e] * scale));
                }
                tmem_st32(t_a + lane_off + c0, a);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(&sm.bar_phiq);
        if (ok) ok = wait_all(&sm.bar_lin, 0);
        if (ok) {
            tc_fence_after();
            const float inv_l = l_eff > 0.0f ? 1.0f / l_eff : 0.0f;
            uint16_t *orow = out + ((size_t)bh * N + (row_valid ? i : 0)) * kD;
#pragma unroll 1
            for (int c0 = 0; c0 < kD; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(o_own + c0, o);
                tmem_wait_ld();
                uint32_t pkk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pkk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
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
        tmem_dealloc(tmem, kAttnTmemCols);
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
    }
    // 16-bit rows of 128 as [64 elements, rows (256 B apart), 2 halves (128 B apart), BH]: a box of
    // {64, 64, 2, 1} lands as the two [64 rows x 128 B] half-tiles one after the other
    const uint64_t dims_h[4] = {64, (uint64_t)g.N, 2, (uint64_t)g.BH};
    const uint64_t st_h[3] = {(uint64_t)kD * 2, 128, (uint64_t)g.N * kD * 2};
    const uint32_t box_h[4] = {64, 64, 2, 1};
    if (!QUANT && !encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, k, dims_h, st_h, box_h))
        return cudaErrorInvalidValue;
    {
        const CUtensorMapDataType vt = QUANT ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        if (!encode_tmap(&tv, vt, 4, v, dims_h, st_h, box_h)) return cudaErrorInvalidValue;
    }
    {
        // H_I^T [128 dims][128 channels] fp32 in rows of kStateCols, viewed as [32 channels, 128 dims
        // (512 B apart), 4 quarters (128 B apart), BH * n_qb]: one box, the four quarter-tiles in order
        const uint64_t hd[4] = {32, (uint64_t)kD, 4, (uint64_t)g.BH * g.n_qb};
        const uint64_t st[3] = {(uint64_t)kD * 4, 128, (uint64_t)kStateCols * 4};
        const uint32_t bh[4] = {32, 128, 4, 1};
        if (!encode_tmap(&th, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, hq, hd, st, bh)) return cudaErrorInvalidValue;
    }
    {
        // raw Q rows of a query block: both 64-channel halves of 128 rows in one box
        const uint32_t bq[4] = {64, 128, 2, 1};
        if (!encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, q, dims_h, st_h, bq)) return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(AttnSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(g.n_qb, g.BH);
    attn_kernel<MODE><<<grid, kAttnThreads, smem, s>>>(tk, tv, th, tq, q8, qscale, kscale, idx, hq, g.N, g.blk_q,
                                                        g.n_qb, g.n_kb, g.k_sel, phi, static_cast<uint16_t *>(out),
                                                        status);
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
