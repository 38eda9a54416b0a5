// sla_ulysses.cu -- layout permutations around the Ulysses all-to-all.
//
// Ulysses context parallelism (the "TurboDiffusion" summary page, 主要能力:
// the training code supports Ulysses CP) keeps, on each of P ranks, a
// contiguous range of n_local = N / P tokens of every head.  Attention needs
// every token of a head, so one all-to-all turns [B, H, n_local, d] (tokens of
// all heads) into [B, H/P, N, d] (all tokens of H/P heads) and another turns the
// attention output back.  Each (batch, head, rank) slice is a contiguous
// n_local x d block in every layout, so the four permutations below move whole
// blocks:
//   mode 0  pack,   tokens -> heads: src [B][H][n][d]          -> dst [P][B][H/P][n][d]
//   mode 1  unpack, tokens -> heads: src [P][B][H/P][n][d]     -> dst [B][H/P][P*n][d]
//   mode 2  pack,   heads -> tokens: src [B][H/P][P*n][d]      -> dst [P][B][H/P][n][d]
//   mode 3  unpack, heads -> tokens: src [P][B][H/P][n][d]     -> dst [B][H][n][d]
// (mode 2 inverts mode 1 and mode 3 inverts mode 0.)  In the send / receive
// buffer [P][B][H/P][n][d], slice r goes to / comes from rank r.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/sla.h"

namespace {

// One CTA per block, indexed in the [P][B][H/P] order of the exchange buffer.
__global__ void __launch_bounds__(256) ulysses_permute_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst,
                                                              int B, int Hp, int P, long long blk_vec, int mode)
{
    const int o = blockIdx.x;  // = (r * B + b) * Hp + hh
    const int hh = o % Hp, b = (o / Hp) % B, r = o / (Hp * B);
    long long seq, buf = (long long)o;
    // block index in the token-sharded layout [B][H] and in the head-sharded layout [B][Hp][P]
    if (mode == 0 || mode == 3) seq = (long long)b * (Hp * P) + (long long)r * Hp + hh;
    else seq = ((long long)b * Hp + hh) * P + r;
    const bool to_buf = (mode == 0 || mode == 2);
    const uint4 *s = src + (to_buf ? seq : buf) * blk_vec;
    uint4 *d = dst + (to_buf ? buf : seq) * blk_vec;
    for (long long i = threadIdx.x; i < blk_vec; i += blockDim.x) d[i] = __ldg(s + i);
}

bool al16(const void *p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" {

sla_status sla_ulysses_permute(const void *src, void *dst, int B, int H, int P, int n_local, int d, int elem_bytes,
                               int mode, void *stream)
{
    if (B < 1 || H < 1 || P < 1 || n_local < 1 || d < 1 || mode < 0 || mode > 3) return SLA_ERR_INVALID_ARG;
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8) return SLA_ERR_INVALID_ARG;
    if (H % P != 0) return SLA_ERR_INVALID_ARG;
    const long long blk_bytes = (long long)n_local * d * elem_bytes;
    if (blk_bytes % 16 != 0) return SLA_ERR_UNSUPPORTED;
    if (!al16(src) || !al16(dst) || src == dst) return SLA_ERR_INVALID_ARG;
    if ((long long)B * H > (1LL << 31) - 1) return SLA_ERR_UNSUPPORTED;
    ulysses_permute_kernel<<<(unsigned)(B * H), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), B, H / P, P, blk_bytes / 16, mode);
    return cudaGetLastError() == cudaSuccess ? SLA_OK : SLA_ERR_CUDA;
}

}  // extern "C"
