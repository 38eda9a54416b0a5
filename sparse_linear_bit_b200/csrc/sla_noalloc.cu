// sla_noalloc.cu -- sla_block_mask_noalloc: the block-mask entry point for
// callers that cannot allocate device memory.
//
// sla_block_mask needs scratch memory (block sums, fp64 scores, a status word
// and the state-reduction mask rows) that its callers pass as a workspace.
// Some callers cannot provide one: code that runs where no allocation may
// happen (inside a framework that owns the whole device-memory budget and
// hands out no raw buffers, or on a latency-critical path where cudaMalloc's
// implicit device synchronisation is not acceptable).  This variant keeps its
// scratch in one file-scope device array of fixed size instead, resident on
// every GPU that loads the library until the process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/sla.h"
#include "sla_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB per device

__device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

// Device address of g_scratch per device.  In host code `g_scratch` names a
// host-side stand-in, so the address must come from cudaGetSymbolAddress with
// that device current.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

void *scratch_for_current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" {

size_t sla_block_mask_noalloc_limit(void) { return kStaticScratchBytes; }

sla_status sla_block_mask_noalloc(const void *q, const void *k, int B, int H, int N, int d, int blk_q, int blk_k,
                                  float topk, int32_t *idx_out, uint32_t *bitmap_out, void *stream)
{
    // the checks of sla_block_mask, in the same order, minus the workspace
    sla_status st = sla::check_shape(B, H, N, d, blk_q, blk_k, topk);
    if (st != SLA_OK) return st;
    const sla::Geometry g = sla::make_geometry(B, H, N, d, blk_q, blk_k, topk, 0);
    auto misaligned = [](const void *p, uintptr_t a) { return p == nullptr || ((uintptr_t)p & (a - 1)) != 0; };
    if (misaligned(q, 16) || misaligned(k, 16)) return SLA_ERR_INVALID_ARG;
    if (g.k_sel > 0 && misaligned(idx_out, 4)) return SLA_ERR_INVALID_ARG;
    if (bitmap_out && ((uintptr_t)bitmap_out & 3u)) return SLA_ERR_INVALID_ARG;
    // scratch regions of the mask path only, each rounded up to 256 bytes: fp64 block means of
    // Q and K, fp64 scores, the mask rows the top-k kernel also writes, and (k_sel == 0 only)
    // a stand-in for the empty index lists
    const size_t BH = (size_t)g.BH;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) / 256 * 256; return o; };
    const size_t o_qbar = take(BH * g.n_qb * sla::kD * sizeof(double));
    const size_t o_kbar = take(BH * g.n_kb * sla::kD * sizeof(double));
    const size_t o_scores = take(BH * g.n_qb * g.n_kb * sizeof(double));
    const size_t o_amask = take(BH * g.n_qb * (size_t)g.n_aw * sizeof(uint32_t));
    const size_t o_idx = g.k_sel > 0 ? 0 : take(BH * g.n_qb * sizeof(int32_t));
    if (off > kStaticScratchBytes) return SLA_ERR_WORKSPACE;  // problem too large for the static scratch
    char *scratch = static_cast<char *>(scratch_for_current_device());
    if (!scratch) return SLA_ERR_CUDA;
    // the mask stages of the forward, with their scratch in the static array
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    double *qbar = reinterpret_cast<double *>(scratch + o_qbar);
    double *kbar = reinterpret_cast<double *>(scratch + o_kbar);
    double *scores = reinterpret_cast<double *>(scratch + o_scores);
    int32_t *idx = g.k_sel > 0 ? idx_out : reinterpret_cast<int32_t *>(scratch + o_idx);
    uint32_t *amask = reinterpret_cast<uint32_t *>(scratch + o_amask);
    if (sla::launch_pool(q, g.BH, N, blk_q, g.n_qb, qbar, nullptr, s) != cudaSuccess) return SLA_ERR_CUDA;
    if (sla::launch_pool(k, g.BH, N, blk_k, g.n_kb, kbar, nullptr, s) != cudaSuccess) return SLA_ERR_CUDA;
    if (sla::launch_scores(qbar, kbar, g, scores, s) != cudaSuccess) return SLA_ERR_CUDA;
    if (sla::launch_topk(scores, g, idx, bitmap_out, amask, s) != cudaSuccess) return SLA_ERR_CUDA;
    return SLA_OK;
}

}  // extern "C"
