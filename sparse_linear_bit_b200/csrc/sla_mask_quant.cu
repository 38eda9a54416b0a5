// sla_mask_quant.cu -- block pooling, fp64 block scores, top-k block
// selection and the smooth-and-quantise step of the SageSLA forward.
//
// * Pooling sums each block's bf16 rows in fp64 and divides by the block's
//   token count once.  Sums of up to 2^17 bf16 values are exact in fp64 unless
//   one (batch, head, channel) spans more than ~2^29 in magnitude, so block
//   sums (and the per-channel mean used for smoothing, summed from per-CTA
//   partial sums) do not depend on the summation order.
// * The score of key block J for query block I is the dot product of their
//   mean rows in fp64, accumulated in channel order with one fused
//   multiply-add per channel ("TurboDiffusion技术架构解析" §2.1: SLA keeps the
//   top-k% most important key-value pairs; the pooled dot product is the
//   importance criterion here).  Identical blocks therefore get identical
//   scores, and ties go to the lower block index.
// * Top-k selection per query block is a radix select on order-preserving
//   64-bit keys of the scores, followed by an in-order pass that takes the
//   lowest-index blocks among those equal to the threshold.
// * Quantisation follows SageAttention's recipe ("清华开源TurboDiffusion加速
//   框架", SageAttention与稀疏计算: FP16 -> INT8): K minus its per-channel mean,
//   one fp32 scale per block (amax / 127), round-to-nearest-even codes clamped
//   to [-127, 127]; each step is one IEEE fp32 operation.
#include <cuda_bf16.h>
#include <cstdint>

#include "sla_internal.h"

namespace sla {
namespace {

// two fp32 -> packed fp8 e4m3 (lo in the low byte), round to nearest even, saturating at +-448
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float (&f)[8])
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// ---------------------------------------------------------------------------
// pooling: mean[bh][J][c] = (sum over the valid rows of block J of x[bh][t][c]) / count,
// and optionally part[bh][chunk][c] = the sum of the block sums of the kPoolBlocks
// blocks this CTA pools (for the per-channel mean over all tokens).
// grid (ceil(nb/kPoolBlocks), BH), 256 threads; thread = (row lane, 8-channel group)
// ---------------------------------------------------------------------------
constexpr int kPoolBlocks = 8;

__global__ void __launch_bounds__(256) pool_kernel(const uint4 *__restrict__ x, int N, int blk, int nb,
                                                   double *__restrict__ mean, double *__restrict__ part)
{
    __shared__ double red[16][kD];
    const int bh = blockIdx.y;
    const int cg = threadIdx.x & 15, rl = threadIdx.x >> 4;
    const uint4 *xh = x + (size_t)bh * N * (kD / 8);
    double total = 0.0;  // thread c < kD: sum of this CTA's block sums of channel c
    for (int J = blockIdx.x * kPoolBlocks; J < min(nb, (blockIdx.x + 1) * kPoolBlocks); ++J) {
        const int t0 = J * blk, t1 = min(N, t0 + blk);
        double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 4
        for (int r = t0 + rl; r < t1; r += 16) {
            float f[8];
            bf16x8_to_f32(__ldg(xh + (size_t)r * (kD / 8) + cg), f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += (double)f[i];
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) red[rl][cg * 8 + i] = acc[i];
        __syncthreads();
        if (threadIdx.x < kD) {
            double sum = 0.0;
#pragma unroll
            for (int r = 0; r < 16; ++r) sum += red[r][threadIdx.x];
            mean[((size_t)bh * nb + J) * kD + threadIdx.x] = sum / (double)(t1 - t0);
            total += sum;
        }
        __syncthreads();
    }
    if (part && threadIdx.x < kD) part[((size_t)bh * gridDim.x + blockIdx.x) * kD + threadIdx.x] = total;
}

// kmean[bh][c] = fp32( (sum of the pooling partial sums of channel c) / N )
__global__ void kmean_kernel(const double *__restrict__ part, int n_parts, int N, float *__restrict__ kmean)
{
    const int bh = blockIdx.x, c = threadIdx.x;
    const double *p = part + (size_t)bh * n_parts * kD + c;
    double s = 0.0;
#pragma unroll 8
    for (int i = 0; i < n_parts; ++i) s += p[(size_t)i * kD];
    kmean[(size_t)bh * kD + c] = (float)(s / (double)N);
}

// ---------------------------------------------------------------------------
// scores[bh][I][J] = fma chain over channels c = 0..127 of qbar[I][c] * kbar[J][c]
// 128 (I) x 64 (J) output tile per CTA; 256 threads as 16 x 16, each 8 x 4
// outputs at rows 2*ty + {0,1} + 32m (m < 4) and columns 2*tx + {0,1} + 32n
// (n < 2), so each operand read is one 16-byte shared load serving two outputs.
// At most 128 registers, so two CTAs share an SM and one's loads overlap the
// other's FMAs.  Channels are staged 16 at a time, transposed to [channel][row].
// ---------------------------------------------------------------------------
constexpr int kScI = 128;
constexpr int kScJ = 64;
constexpr int kScChan = 16;

__global__ void __launch_bounds__(256, 2) scores_kernel(const double *__restrict__ qbar,
                                                        const double *__restrict__ kbar, int n_qb, int n_kb,
                                                        double *__restrict__ scores)
{
    __shared__ __align__(16) double As[kScChan][kScI];
    __shared__ __align__(16) double Bs[kScChan][kScJ];
    const int bh = blockIdx.z, I0 = blockIdx.y * kScI, J0 = blockIdx.x * kScJ;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const double *qh = qbar + (size_t)bh * n_qb * kD;
    const double *kh = kbar + (size_t)bh * n_kb * kD;
    double acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int c0 = 0; c0 < kD; c0 += kScChan) {
        // thread -> (row = e & 127, channel pair = e >> 7): consecutive threads store consecutive
        // rows of one channel (no bank conflicts); B covers 64 rows with the same mapping
#pragma unroll
        for (int l = 0; l < 4; ++l) {
            const int e = tid + 256 * l, r = e & 127, c = 2 * (e >> 7);
            double2 a = make_double2(0.0, 0.0);
            if (I0 + r < n_qb) a = __ldg(reinterpret_cast<const double2 *>(qh + (size_t)(I0 + r) * kD + c0 + c));
            As[c][r] = a.x;
            As[c + 1][r] = a.y;
        }
#pragma unroll
        for (int l = 0; l < 2; ++l) {
            const int e = tid + 256 * l, r = e & 63, c = 2 * (e >> 6);
            double2 b = make_double2(0.0, 0.0);
            if (J0 + r < n_kb) b = __ldg(reinterpret_cast<const double2 *>(kh + (size_t)(J0 + r) * kD + c0 + c));
            Bs[c][r] = b.x;
            Bs[c + 1][r] = b.y;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < kScChan; ++c) {
            double a[8], b[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const double2 av = *reinterpret_cast<const double2 *>(&As[c][2 * ty + 32 * m]);
                a[2 * m] = av.x;
                a[2 * m + 1] = av.y;
            }
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                const double2 bv = *reinterpret_cast<const double2 *>(&Bs[c][2 * tx + 32 * n]);
                b[2 * n] = bv.x;
                b[2 * n + 1] = bv.y;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    double *sh = scores + (size_t)bh * n_qb * n_kb;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int I = I0 + 2 * ty + (i & 1) + 32 * (i >> 1);
        if (I >= n_qb) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int J = J0 + 2 * tx + (j & 1) + 32 * (j >> 1);
            if (J < n_kb) sh[(size_t)I * n_kb + J] = acc[i][j] + 0.0;  // -0 -> +0
        }
    }
}

// ---------------------------------------------------------------------------
// top-k selection: one CTA (128 threads) per (bh, I)
// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 128;

__device__ __forceinline__ uint64_t order_key(double s)
{
    const uint64_t u = (uint64_t)__double_as_longlong(s);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// exclusive prefix sum over the CTA (128 threads); returns the total in *total
__device__ int block_exclusive_scan(int v, int *total, int *warp_tmp)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tmp[w] = x;
    __syncthreads();
    int base = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < kTopkThreads / 32; ++i) {
        if (i < w) base += warp_tmp[i];
        tot += warp_tmp[i];
    }
    __syncthreads();
    *total = tot;
    return base + x - v;
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const double *__restrict__ scores, int n_qb, int n_kb,
                                                            int n_aw, int k_sel, int subtract,
                                                            int32_t *__restrict__ idx, uint32_t *__restrict__ bitmap,
                                                            uint32_t *__restrict__ amask)
{
    extern __shared__ uint64_t keys[];  // [n_kb], then the selection bits [n_aw] (32-bit words)
    __shared__ int hist[256];
    __shared__ int warp_tmp[kTopkThreads / 32];
    __shared__ int s_bin, s_remaining;
    const int row = blockIdx.x;  // bh * n_qb + I
    const double *sr = scores + (size_t)row * n_kb;
    uint32_t *sel_bits = reinterpret_cast<uint32_t *>(keys + n_kb);
    for (int J = threadIdx.x; J < n_kb; J += kTopkThreads) keys[J] = order_key(sr[J]);
    for (int w = threadIdx.x; w < n_aw; w += kTopkThreads) sel_bits[w] = 0u;

    // radix select for the k_sel-th largest key
    uint64_t prefix = 0, mask = 0;
    int remaining = k_sel;
    if (k_sel > 0 && k_sel < n_kb) {
        for (int shift = 56; shift >= 0; shift -= 8) {
            for (int b = threadIdx.x; b < 256; b += kTopkThreads) hist[b] = 0;
            __syncthreads();
            for (int J = threadIdx.x; J < n_kb; J += kTopkThreads) {
                const uint64_t k = keys[J];
                if ((k & mask) == prefix) atomicAdd(&hist[(int)((k >> shift) & 255u)], 1);
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                int cum = 0, b = 255;
                for (; b > 0; --b) {
                    if (cum + hist[b] >= remaining) break;
                    cum += hist[b];
                }
                s_bin = b;
                s_remaining = remaining - cum;
            }
            __syncthreads();
            prefix |= (uint64_t)s_bin << shift;
            mask |= (uint64_t)255u << shift;
            remaining = s_remaining;
            __syncthreads();
        }
    }
    // selected: key > T, or key == T and among the first `remaining` such in J order
    const uint64_t T = prefix;
    const int chunk = (n_kb + kTopkThreads - 1) / kTopkThreads;
    const int j0 = min(n_kb, threadIdx.x * chunk), j1 = min(n_kb, j0 + chunk);
    auto base_sel = [&](int J) -> int {
        if (k_sel == 0) return 0;
        if (k_sel >= n_kb) return 1;
        return keys[J] > T ? 1 : 0;
    };
    int n_eq = 0;
    if (k_sel > 0 && k_sel < n_kb)
        for (int J = j0; J < j1; ++J) n_eq += (keys[J] == T);
    int tot;
    const int eq_before = block_exclusive_scan(n_eq, &tot, warp_tmp);
    int n_sel = 0, e = eq_before;
    for (int J = j0; J < j1; ++J) {
        int s = base_sel(J);
        if (!s && k_sel > 0 && k_sel < n_kb && keys[J] == T) s = (e++ < remaining);
        n_sel += s;
    }
    const int sel_before = block_exclusive_scan(n_sel, &tot, warp_tmp);
    // write the ascending index list; gather the selection bits in shared memory
    int32_t *ir = idx + (size_t)row * k_sel;
    int o = sel_before;
    e = eq_before;
    uint32_t word = 0;
    int cur_w = j0 >> 5;
    for (int J = j0; J < j1; ++J) {
        int s = base_sel(J);
        if (!s && k_sel > 0 && k_sel < n_kb && keys[J] == T) s = (e++ < remaining);
        if (s) ir[o++] = J;
        if ((J >> 5) != cur_w) {
            if (word) atomicOr(&sel_bits[cur_w], word);
            word = 0;
            cur_w = J >> 5;
        }
        if (s) word |= 1u << (J & 31);
    }
    if (word) atomicOr(&sel_bits[cur_w], word);
    __syncthreads();
    // the bitmap (selected) and the state-reduction mask row (selected, or its valid complement)
    const int words = (n_kb + 31) / 32;
    uint32_t *br = bitmap ? bitmap + (size_t)row * words : nullptr;
    uint32_t *ar = amask + (size_t)row * n_aw;
    for (int w = threadIdx.x; w < n_aw; w += kTopkThreads) {
        const uint32_t sb = sel_bits[w];
        const int valid_bits = min(32, max(0, n_kb - 32 * w));
        const uint32_t valid = valid_bits == 32 ? 0xFFFFFFFFu : (1u << valid_bits) - 1u;
        ar[w] = subtract ? sb : (~sb & valid);
        if (br && w < words) br[w] = sb;
    }
}

// ---------------------------------------------------------------------------
// top-k selection, one warp per (bh, I) row, keys in registers (J = 32m + lane).
// Radix select on the order-preserving 64-bit keys, 8 bits per pass, with a
// warp-private shared histogram; after each pass the bin holding the k_sel-th
// largest key is found by a warp suffix scan.  It stops early once every key
// matching the resolved prefix P is selected.  Selected: (key & mask) > P, or
// == P and among the first R such keys in J order (ties to the lower index),
// ranked with ballots.  The bitmap words are the ballots themselves.
// ---------------------------------------------------------------------------
constexpr int kTopkWarps = 4;

template <int KPL>  // keys per lane: n_kb <= 32 * KPL
__global__ void __launch_bounds__(32 * kTopkWarps) topk_warp_kernel(const double *__restrict__ scores, int n_rows,
                                                                    int n_kb, int n_aw, int k_sel, int subtract,
                                                                    int32_t *__restrict__ idx,
                                                                    uint32_t *__restrict__ bitmap,
                                                                    uint32_t *__restrict__ amask)
{
    __shared__ int hist_all[kTopkWarps][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kTopkWarps + warp;
    if (row >= n_rows) return;  // warp-uniform: this kernel has no block-wide synchronisation
    int *hist = hist_all[warp];
    const unsigned lt_mask = (1u << lane) - 1u;
    const double *sr = scores + (size_t)row * n_kb;
    uint64_t key[KPL];
#pragma unroll
    for (int m = 0; m < KPL; ++m) {
        const int J = 32 * m + lane;
        key[m] = J < n_kb ? order_key(__ldg(sr + J)) : 0ull;
    }
    uint64_t P = 0, mask = 0;
    int R = k_sel;
    const bool partial = k_sel > 0 && k_sel < n_kb;
    if (partial) {
        for (int shift = 56; shift >= 0; shift -= 8) {
#pragma unroll
            for (int b = lane; b < 256; b += 32) hist[b] = 0;
            __syncwarp();
#pragma unroll
            for (int m = 0; m < KPL; ++m)
                if (32 * m + lane < n_kb && (key[m] & mask) == P) atomicAdd(&hist[(int)((key[m] >> shift) & 255u)], 1);
            __syncwarp();
            // lane L covers bins 255-8L .. 248-8L (top first); suffix counts by an inclusive lane scan
            const int top = 255 - 8 * lane;
            int h8[8], tot = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                h8[e] = hist[top - e];
                tot += h8[e];
            }
            int incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int L = __ffs(__ballot_sync(0xffffffffu, incl >= R)) - 1;  // candidates >= R, so L >= 0
            int bsel = 0, rn = 0, cnt = 0;
            if (lane == L) {
                int cum = incl - tot;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (cnt == 0 && cum + h8[e] >= R) {
                        bsel = top - e;
                        rn = R - cum;
                        cnt = h8[e];
                    }
                    cum += h8[e];
                }
            }
            bsel = __shfl_sync(0xffffffffu, bsel, L);
            rn = __shfl_sync(0xffffffffu, rn, L);
            cnt = __shfl_sync(0xffffffffu, cnt, L);
            P |= (uint64_t)bsel << shift;
            mask |= (uint64_t)255u << shift;
            R = rn;
            __syncwarp();  // every lane has read the histogram before the next pass clears it
            if (cnt == R) break;  // every key matching P is selected
        }
    }
    int32_t *ir = idx + (size_t)row * k_sel;
    uint32_t *ar = amask + (size_t)row * n_aw;
    uint32_t *br = bitmap ? bitmap + (size_t)row * ((n_kb + 31) / 32) : nullptr;
    int o = 0, eq_seen = 0;
#pragma unroll
    for (int m = 0; m < KPL; ++m) {
        if (32 * m >= n_kb) break;  // warp-uniform
        const int J = 32 * m + lane;
        const bool valid = J < n_kb;
        bool s;
        if (!partial) {
            s = valid && k_sel > 0;
        } else {
            const uint64_t km = key[m] & mask;
            const bool eq = valid && km == P;
            const unsigned eqb = __ballot_sync(0xffffffffu, eq);
            s = (valid && km > P) || (eq && eq_seen + __popc(eqb & lt_mask) < R);
            eq_seen += __popc(eqb);
        }
        const unsigned sb = __ballot_sync(0xffffffffu, s);
        const unsigned ab = __ballot_sync(0xffffffffu, valid && (s != (subtract == 0)));
        if (s) ir[o + __popc(sb & lt_mask)] = J;
        o += __popc(sb);
        if (lane == 0) {
            ar[m] = ab;
            if (br) br[m] = sb;
        }
    }
    for (int w = (n_kb + 31) / 32 + lane; w < n_aw; w += 32) ar[w] = 0u;  // the last k-step's padding
}

// ---------------------------------------------------------------------------
// quantisation: one CTA per block, 256 threads; SMOOTH subtracts mean[c].
// The block stays in registers as packed bf16 (the values are re-expanded for
// the second pass), which keeps the kernel at full occupancy.
//
// Codes: c = clamp(rint(fl(x / s)), -127, 127) with fl the IEEE fp32 quotient.
// Instead of a division per element, t = fl(x * r) with r = fl(1 / s) is
// used: |t - x/s| <= |x/s| (2^-24 + 2^-24 + 2^-48) and |fl(x/s) - x/s| <=
// |x/s| 2^-24, so for |x/s| <= 128 (|x| <= amax = 127 s, up to rounding)
// |t - fl(x/s)| < 2.3e-5.  Unless t lies within 2^-14 of a half-integer, no
// rounding boundary of rint separates t from fl(x/s) and rint(t) is the
// code; otherwise (about 1 element in 8000) the IEEE quotient is taken.  On
// the fast path |t| <= 127 (1 + 3 * 2^-24), so rint(t) needs no clamp, and the
// low byte of the bits of t + 1.5 * 2^23 (which rounds t to an integer, ties to
// even) is rint(t) in two's complement.
//
// FP8 (e4m3) codes: s = amax / 448 and code = e4m3(fl(x / s)), round to nearest
// even with saturation (an added mode: the pages name INT8/INT4 only).  The same
// reciprocal product is used; |t - fl(x/s)| < 2^-22 |t|, so when t (1 - 2^-20)
// and t (1 + 2^-20) convert to the same code it is the quotient's code.
// ---------------------------------------------------------------------------
// When `bmean` is given (Q only), the kernel also writes the block's fp64 mean
// row, the pooled mean that block selection scores with (exact fp64 sums, so the
// same values as the pooling kernel's).
template <bool SMOOTH, int BLK, bool FP8>
__global__ void __launch_bounds__(256) quant_kernel(const uint4 *__restrict__ x, int N, int nb,
                                                    const float *__restrict__ mean, uint2 *__restrict__ out,
                                                    float *__restrict__ scale, double *__restrict__ bmean)
{
    constexpr int kVec = BLK * (kD / 8) / 256;  // uint4 per thread
    __shared__ float warp_max[8];
    __shared__ double part[8][16][8];  // block-mean partials: [warp][channel group][channel]
    const int bh = blockIdx.y, J = blockIdx.x;
    const int t0 = J * BLK;
    const int rows = min(BLK, N - t0);
    const int cg = threadIdx.x & 15;  // the thread's 8-channel group (same for every l)
    const uint4 *xb = x + ((size_t)bh * N + t0) * (kD / 8);
    float mu[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) mu[i] = SMOOTH ? __ldg(mean + (size_t)bh * kD + cg * 8 + i) : 0.0f;
    uint4 raw[kVec];
#pragma unroll
    for (int l = 0; l < kVec; ++l) {
        const int e = threadIdx.x + 256 * l;  // uint4 index within block: row = e/16, chunk = e%16
        raw[l] = (e >> 4) < rows ? __ldg(xb + e) : make_uint4(0, 0, 0, 0);
    }
    auto expand = [&](const uint4 &u, float (&f)[8]) {
        bf16x8_to_f32(u, f);
        if (SMOOTH) {
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = __fsub_rn(f[i], mu[i]);
        }
    };
    float amax = 0.0f;
    double bsum[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int l = 0; l < kVec; ++l) {
        if (((threadIdx.x + 256 * l) >> 4) < rows) {
            float f[8];
            expand(raw[l], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
            if (!SMOOTH && bmean) {  // without smoothing f holds the raw values
#pragma unroll
                for (int i = 0; i < 8; ++i) bsum[i] += (double)f[i];
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
    if (!SMOOTH && bmean) {  // lanes cg and cg + 16 of a warp share a channel group
#pragma unroll
        for (int i = 0; i < 8; ++i) bsum[i] += __shfl_xor_sync(0xffffffffu, bsum[i], 16);
        if ((threadIdx.x & 31) < 16) {
#pragma unroll
            for (int i = 0; i < 8; ++i) part[threadIdx.x >> 5][cg][i] = bsum[i];
        }
    }
    __syncthreads();
    if (!SMOOTH && bmean && threadIdx.x < kD) {
        const int c = threadIdx.x;
        double sum = 0.0;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += part[w][c >> 3][c & 7];
        bmean[((size_t)bh * nb + J) * kD + c] = sum / (double)rows;
    }
    amax = warp_max[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, warp_max[w]);
    const float s = __fdiv_rn(amax, FP8 ? 448.0f : 127.0f);
    if (threadIdx.x == 0) scale[(size_t)bh * nb + J] = s;
    const float r = s != 0.0f ? __fdiv_rn(1.0f, s) : 0.0f;
    const bool fast = s != 0.0f && isfinite(r);
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: t + kRound rounds t to an integer (ties to even)
    uint2 *ob = out + ((size_t)bh * N + t0) * (kD / 8);
#pragma unroll
    for (int l = 0; l < kVec; ++l) {
        const int e = threadIdx.x + 256 * l;
        if ((e >> 4) < rows) {
            float f[8];
            expand(raw[l], f);
            uint32_t w0, w1;
            if (FP8) {
                // The e4m3 code of t = fl(x * r) is that of the IEEE quotient unless a rounding
                // boundary of e4m3 lies within 2^-22 |t| of t (see above): t (1 -+ 2^-20) bracket
                // that interval, so equal codes at both ends settle it.
                uint32_t c[4], slow = fast ? 0u : 0xFu;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float t0 = f[2 * i] * r, t1 = f[2 * i + 1] * r;
                    const uint32_t lo = e4m3x2(t0 * (1.0f - 9.5367431640625e-07f), t1 * (1.0f - 9.5367431640625e-07f));
                    const uint32_t hi = e4m3x2(t0 * (1.0f + 9.5367431640625e-07f), t1 * (1.0f + 9.5367431640625e-07f));
                    if (lo != hi) slow |= 1u << i;
                    c[i] = lo;
                }
                if (slow) {  // rare: near an e4m3 rounding boundary, or a zero / tiny scale
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (slow & (1u << i))
                            c[i] = s != 0.0f ? e4m3x2(__fdiv_rn(f[2 * i], s), __fdiv_rn(f[2 * i + 1], s)) : 0u;
                }
                w0 = c[0] | (c[1] << 16);
                w1 = c[2] | (c[3] << 16);
            } else {
                // fast path: the low byte of the bits of t + kRound is rint(t) as int8 (|t| <= 127 here)
                uint32_t cb[8];
                unsigned slow = fast ? 0u : 0xFFu;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float t = f[i] * r;
                    const float qf = __fadd_rn(t, kRound);
                    const float rt = __fsub_rn(qf, kRound);
                    if (fabsf(t - rt) > 0.5f - 6.103515625e-05f) slow |= 1u << i;
                    cb[i] = __float_as_uint(qf);
                }
                if (slow) {  // rare: within 2^-14 of a half-integer, or a zero / tiny scale
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (slow & (1u << i)) {
                            int c = 0;
                            if (s != 0.0f) c = max(-127, min(127, __float2int_rn(__fdiv_rn(f[i], s))));
                            cb[i] = (uint32_t)c;
                        }
                    }
                }
                w0 = __byte_perm(__byte_perm(cb[0], cb[1], 0x0040), __byte_perm(cb[2], cb[3], 0x0040), 0x5410);
                w1 = __byte_perm(__byte_perm(cb[4], cb[5], 0x0040), __byte_perm(cb[6], cb[7], 0x0040), 0x5410);
            }
            ob[e] = make_uint2(w0, w1);
        }
    }
}

}  // namespace

int pool_parts(int nb) { return (nb + kPoolBlocks - 1) / kPoolBlocks; }

cudaError_t launch_pool(const void *x, int BH, int N, int blk, int nb, double *mean, double *part, cudaStream_t s)
{
    dim3 grid(pool_parts(nb), BH);
    pool_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4 *>(x), N, blk, nb, mean, part);
    return cudaGetLastError();
}

cudaError_t launch_kmean(const double *part, int BH, int N, int n_parts, float *kmean, cudaStream_t s)
{
    kmean_kernel<<<BH, kD, 0, s>>>(part, n_parts, N, kmean);
    return cudaGetLastError();
}

cudaError_t launch_scores(const double *qbar, const double *kbar, const Geometry &g, double *scores, cudaStream_t s)
{
    dim3 grid((g.n_kb + kScJ - 1) / kScJ, (g.n_qb + kScI - 1) / kScI, g.BH);
    scores_kernel<<<grid, 256, 0, s>>>(qbar, kbar, g.n_qb, g.n_kb, scores);
    return cudaGetLastError();
}

cudaError_t launch_topk(const double *scores, const Geometry &g, int32_t *idx, uint32_t *bitmap, uint32_t *amask,
                        cudaStream_t s)
{
    const int rows = g.BH * g.n_qb;
    const unsigned blocks = (unsigned)((rows + kTopkWarps - 1) / kTopkWarps);
    const int sub = g.subtract ? 1 : 0;
    // one warp per row while the row's keys fit in registers
    if (g.n_kb <= 32 * 8) {
        topk_warp_kernel<8><<<blocks, 32 * kTopkWarps, 0, s>>>(scores, rows, g.n_kb, g.n_aw, g.k_sel, sub, idx,
                                                               bitmap, amask);
        return cudaGetLastError();
    }
    if (g.n_kb <= 32 * 40) {
        topk_warp_kernel<40><<<blocks, 32 * kTopkWarps, 0, s>>>(scores, rows, g.n_kb, g.n_aw, g.k_sel, sub, idx,
                                                                bitmap, amask);
        return cudaGetLastError();
    }
    const size_t smem = sizeof(uint64_t) * (size_t)g.n_kb + sizeof(uint32_t) * (size_t)g.n_aw;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    topk_kernel<<<rows, kTopkThreads, smem, s>>>(scores, g.n_qb, g.n_kb, g.n_aw, g.k_sel, sub, idx, bitmap, amask);
    return cudaGetLastError();
}

cudaError_t launch_quant(const void *x, int BH, int N, int blk, int nb, const float *mean, int8_t *out, float *scale,
                         double *bmean, int fp8, cudaStream_t s)
{
    dim3 grid(nb, BH);
    const uint4 *xi = static_cast<const uint4 *>(x);
    uint2 *o = reinterpret_cast<uint2 *>(out);
    if (mean) {
        if (blk != 64 || bmean) return cudaErrorInvalidValue;
        if (fp8) quant_kernel<true, 64, true><<<grid, 256, 0, s>>>(xi, N, nb, mean, o, scale, nullptr);
        else quant_kernel<true, 64, false><<<grid, 256, 0, s>>>(xi, N, nb, mean, o, scale, nullptr);
    } else if (blk == 128) {
        if (fp8) quant_kernel<false, 128, true><<<grid, 256, 0, s>>>(xi, N, nb, nullptr, o, scale, bmean);
        else quant_kernel<false, 128, false><<<grid, 256, 0, s>>>(xi, N, nb, nullptr, o, scale, bmean);
    } else if (blk == 64) {
        if (fp8) quant_kernel<false, 64, true><<<grid, 256, 0, s>>>(xi, N, nb, nullptr, o, scale, bmean);
        else quant_kernel<false, 64, false><<<grid, 256, 0, s>>>(xi, N, nb, nullptr, o, scale, bmean);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace sla
