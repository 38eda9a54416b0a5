// sla_api.cu -- the C ABI of libsla.so (declared in include/sla.h): argument
// validation, workspace layout and the launch sequence of the SageSLA forward.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/sla.h"

#include "sla_internal.h"

namespace sla {

int topk_count(int n_kb, float topk)
{
    if (n_kb < 0 || !(topk >= 0.0f && topk <= 1.0f)) return -1;
    double x = std::floor((double)topk * (double)n_kb + 1e-4);
    if (x < 0.0) x = 0.0;
    if (x > (double)n_kb) x = (double)n_kb;
    return (int)x;
}

Geometry make_geometry(int B, int H, int N, int d, int blk_q, int blk_k, float topk, int quant)
{
    Geometry g{};
    g.B = B; g.H = H; g.N = N; g.d = d; g.blk_q = blk_q; g.blk_k = blk_k; g.quant = quant;
    g.BH = B * H;
    g.n_qb = (N + blk_q - 1) / blk_q;
    g.n_kb = (N + blk_k - 1) / blk_k;
    g.n_aw = 2 * ((g.n_kb + 63) / 64);  // whole 64-block k-steps of the state reduction
    g.k_sel = topk_count(g.n_kb, topk);
    g.subtract = 2 * g.k_sel <= g.n_kb;
    g.n_chunks = (g.n_kb + kStateChunk - 1) / kStateChunk;
    return g;
}

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

Layout make_layout(const Geometry &g)
{
    Layout L{};
    const size_t BH = (size_t)g.BH, N = (size_t)g.N;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
    L.status = take(256);
    L.qbar = take(BH * g.n_qb * kD * sizeof(double));
    L.kbar = take(BH * g.n_kb * kD * sizeof(double));
    L.kpart = take(BH * (size_t)pool_parts(g.n_kb) * kD * sizeof(double));
    L.scores = take(BH * g.n_qb * g.n_kb * sizeof(double));
    L.idx = take(BH * g.n_qb * (size_t)(g.k_sel > 0 ? g.k_sel : 1) * sizeof(int32_t));
    L.amask = take(BH * g.n_qb * (size_t)g.n_aw * sizeof(uint32_t));
    const size_t none = (size_t)-1;
    L.q8 = g.quant ? take(BH * N * kD) : none;
    L.k8 = g.quant ? take(BH * N * kD) : none;
    L.qscale = g.quant ? take(BH * g.n_qb * sizeof(float)) : none;
    L.kscale = g.quant ? take(BH * g.n_kb * sizeof(float)) : none;
    L.kmean = take(BH * kD * sizeof(float));
    L.states = take(BH * g.n_kb * (size_t)kStateCols * sizeof(uint16_t));
    L.partials = take(BH * g.n_chunks * (size_t)kStateCols * sizeof(float));
    L.htot = take(BH * (size_t)kStateCols * sizeof(float));
    L.hq = take(BH * g.n_qb * (size_t)kStateCols * sizeof(float));
    L.v16 = g.quant ? none : take(BH * N * kD * sizeof(uint16_t));
    L.total = off;
    return L;
}

// ---------------------------------------------------------------------------
// TMA descriptor encoding through the driver entry point
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

bool encode_tmap(CUtensorMap *map, CUtensorMapDataType dtype, int rank, const void *base, const uint64_t *dims,
                 const uint64_t *strides_bytes, const uint32_t *box)
{
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return false;
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i < rank - 1) st[i] = strides_bytes[i];
    }
    CUresult r = g_encode(map, dtype, (cuuint32_t)rank, const_cast<void *>(base), d, st, bx, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace sla

using namespace sla;

namespace {

bool aligned16(const void *p) { return p && ((uintptr_t)p & 15u) == 0; }

char *ws_at(void *ws, size_t off) { return static_cast<char *>(ws) + off; }

#define SLA_TRY(expr)                                                    \
    do {                                                                 \
        cudaError_t _e = (expr);                                         \
        if (_e != cudaSuccess) return SLA_ERR_CUDA;                      \
    } while (0)

}  // namespace

namespace sla {

// shared validation of (B, H, N, d, blk_q, blk_k, topk)
sla_status check_shape(int B, int H, int N, int d, int blk_q, int blk_k, float topk)
{
    if (B < 1 || H < 1 || N < 1 || d < 1 || blk_q < 1 || blk_k < 1) return SLA_ERR_INVALID_ARG;
    if (!(topk >= 0.0f && topk <= 1.0f)) return SLA_ERR_INVALID_ARG;
    if ((long long)B * H > (1LL << 24) || (long long)N > (1LL << 24)) return SLA_ERR_UNSUPPORTED;
    if (d != kD || blk_k != kBlkK || (blk_q != 64 && blk_q != 128)) return SLA_ERR_UNSUPPORTED;
    // int8 logits are converted exactly through a 2^22 window; the top-k kernel keeps one
    // row of 64-bit keys in shared memory
    if ((N + blk_k - 1) / blk_k > 24576) return SLA_ERR_UNSUPPORTED;
    return SLA_OK;
}

sla_status quantize_qk(const void *q, const void *k, int B, int H, int N, int d, int blk_q, int blk_k, int fp8,
                           int8_t *q_i8, int8_t *k_i8, float *q_scale, float *k_scale, float *k_mean, void *ws,
                           size_t ws_bytes, void *stream)
{
    sla_status st = check_shape(B, H, N, d, blk_q, blk_k, 0.0f);
    if (st != SLA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(ws) || !aligned16(q_i8) || !aligned16(k_i8))
        return SLA_ERR_INVALID_ARG;
    if (!q_scale || !k_scale || ((uintptr_t)q_scale & 3u) || ((uintptr_t)k_scale & 3u) ||
        (k_mean && ((uintptr_t)k_mean & 3u)))
        return SLA_ERR_INVALID_ARG;
    const Geometry g = make_geometry(B, H, N, d, blk_q, blk_k, 0.0f, 1);
    const Layout L = make_layout(g);
    if (ws_bytes < L.total) return SLA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    SLA_TRY(cudaMemsetAsync(ws_at(ws, L.status), 0, sizeof(int), s));
    double *kbar = reinterpret_cast<double *>(ws_at(ws, L.kbar));
    double *kpart = reinterpret_cast<double *>(ws_at(ws, L.kpart));
    float *mean = k_mean ? k_mean : reinterpret_cast<float *>(ws_at(ws, L.kmean));
    SLA_TRY(launch_pool(k, g.BH, N, blk_k, g.n_kb, kbar, kpart, s));
    SLA_TRY(launch_kmean(kpart, g.BH, N, pool_parts(g.n_kb), mean, s));
    SLA_TRY(launch_quant(q, g.BH, N, blk_q, g.n_qb, nullptr, q_i8, q_scale, nullptr, fp8, s));
    SLA_TRY(launch_quant(k, g.BH, N, blk_k, g.n_kb, mean, k_i8, k_scale, nullptr, fp8, s));
    return SLA_OK;
}
}  // namespace sla

extern "C" {

const char *sla_version(void) { return "sla-b200 0.1.0 (sm_100a)"; }

const char *sla_status_string(int status)
{
    switch (status) {
    case SLA_OK: return "SLA_OK";
    case SLA_ERR_INVALID_ARG: return "SLA_ERR_INVALID_ARG";
    case SLA_ERR_UNSUPPORTED: return "SLA_ERR_UNSUPPORTED";
    case SLA_ERR_WORKSPACE: return "SLA_ERR_WORKSPACE";
    case SLA_ERR_CUDA: return "SLA_ERR_CUDA";
    case SLA_ERR_TIMEOUT: return "SLA_ERR_TIMEOUT";
    default: return "SLA_ERR_UNKNOWN";
    }
}

int sla_topk_count(int n_kb, float topk) { return topk_count(n_kb, topk); }

size_t sla_workspace_bytes(int B, int H, int N, int d, int blk_q, int blk_k, float topk, int quant)
{
    if (check_shape(B, H, N, d, blk_q, blk_k, topk) != SLA_OK || quant < 0 || quant > 2) return 0;
    return make_layout(make_geometry(B, H, N, d, blk_q, blk_k, topk, quant)).total;
}

int sla_workspace_layout(int B, int H, int N, int d, int blk_q, int blk_k, float topk, int quant, size_t *offsets,
                         int n)
{
    if (check_shape(B, H, N, d, blk_q, blk_k, topk) != SLA_OK || quant < 0 || quant > 2) return 0;
    const Layout L = make_layout(make_geometry(B, H, N, d, blk_q, blk_k, topk, quant));
    const size_t v[17] = {L.status, L.qbar,  L.kbar,   L.scores,   L.idx,  L.amask, L.q8,  L.k8,   L.qscale,
                          L.kscale, L.kmean, L.states, L.partials, L.htot, L.hq,    L.v16, L.kpart};
    for (int i = 0; i < n && i < 17; ++i) offsets[i] = v[i];
    return 17;
}

sla_status sla_block_mask(const void *q, const void *k, int B, int H, int N, int d, int blk_q, int blk_k, float topk,
                          int32_t *idx_out, uint32_t *bitmap_out, void *ws, size_t ws_bytes, void *stream)
{
    sla_status st = check_shape(B, H, N, d, blk_q, blk_k, topk);
    if (st != SLA_OK) return st;
    const Geometry g = make_geometry(B, H, N, d, blk_q, blk_k, topk, 0);
    if (!aligned16(q) || !aligned16(k) || !aligned16(ws)) return SLA_ERR_INVALID_ARG;
    if (g.k_sel > 0 && (!idx_out || ((uintptr_t)idx_out & 3u))) return SLA_ERR_INVALID_ARG;
    if (bitmap_out && ((uintptr_t)bitmap_out & 3u)) return SLA_ERR_INVALID_ARG;
    const Layout L = make_layout(g);
    if (ws_bytes < L.total) return SLA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    SLA_TRY(cudaMemsetAsync(ws_at(ws, L.status), 0, sizeof(int), s));
    double *qbar = reinterpret_cast<double *>(ws_at(ws, L.qbar));
    double *kbar = reinterpret_cast<double *>(ws_at(ws, L.kbar));
    double *scores = reinterpret_cast<double *>(ws_at(ws, L.scores));
    SLA_TRY(launch_pool(q, g.BH, N, blk_q, g.n_qb, qbar, nullptr, s));
    SLA_TRY(launch_pool(k, g.BH, N, blk_k, g.n_kb, kbar, nullptr, s));
    SLA_TRY(launch_scores(qbar, kbar, g, scores, s));
    int32_t *idx = g.k_sel > 0 ? idx_out : reinterpret_cast<int32_t *>(ws_at(ws, L.idx));
    SLA_TRY(launch_topk(scores, g, idx, bitmap_out, reinterpret_cast<uint32_t *>(ws_at(ws, L.amask)), s));
    return SLA_OK;
}

sla_status sla_quantize_qk(const void *q, const void *k, int B, int H, int N, int d, int blk_q, int blk_k,
                           int8_t *q_i8, int8_t *k_i8, float *q_scale, float *k_scale, float *k_mean, void *ws,
                           size_t ws_bytes, void *stream)
{
    return quantize_qk(q, k, B, H, N, d, blk_q, blk_k, 0, q_i8, k_i8, q_scale, k_scale, k_mean, ws, ws_bytes, stream);
}

sla_status sla_quantize_qk_fp8(const void *q, const void *k, int B, int H, int N, int d, int blk_q, int blk_k,
                               uint8_t *q_fp8, uint8_t *k_fp8, float *q_scale, float *k_scale, float *k_mean,
                               void *ws, size_t ws_bytes, void *stream)
{
    return quantize_qk(q, k, B, H, N, d, blk_q, blk_k, 1, reinterpret_cast<int8_t *>(q_fp8),
                       reinterpret_cast<int8_t *>(k_fp8), q_scale, k_scale, k_mean, ws, ws_bytes, stream);
}

}  // extern "C"

namespace {

// A second stream and three events for one forward call; released when the call returns (CUDA
// frees them once the work queued on them has completed).
struct ForkK {
    cudaStream_t st = nullptr;
    cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};  // fork, K block means ready, K side done
    bool make()
    {
        if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return false;
        for (cudaEvent_t &e : ev)
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
        return true;
    }
    ~ForkK()
    {
        for (cudaEvent_t e : ev)
            if (e) cudaEventDestroy(e);
        if (st) cudaStreamDestroy(st);
    }
};

// The forward's launch sequence.  When `ev` is non-null, an event is recorded
// before the first stage and after each of the kStages stages (on `s`), and every
// stage runs on `s` in order.  Otherwise the K side (K's block means and partial
// sums, the linear states and the global state, K's smoothing mean and codes)
// runs on a second stream beside the Q side and the block selection, which need
// from it only the K block means; the two meet before the state reduction.  The
// selection's fp64 scores and top-k then overlap the K side's memory traffic.
constexpr int kProfStages = 7;  // pool, scores+top-k, quantise, states, state reduce, attention, total
sla_status run_forward(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d, int blk_q,
                       int blk_k, float topk, int phi, int quant, void *ws, size_t ws_bytes, cudaStream_t s,
                       cudaEvent_t *ev, bool reset_status = true)
{
    sla_status st = check_shape(B, H, N, d, blk_q, blk_k, topk);
    if (st != SLA_OK) return st;
    if (phi != SLA_PHI_ELU1 && phi != SLA_PHI_RELU) return SLA_ERR_INVALID_ARG;
    if (quant < 0 || quant > 2) return SLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(ws))
        return SLA_ERR_INVALID_ARG;
    const Geometry g = make_geometry(B, H, N, d, blk_q, blk_k, topk, quant);
    const Layout L = make_layout(g);
    if (ws_bytes < L.total) return SLA_ERR_WORKSPACE;
    int *status = reinterpret_cast<int *>(ws_at(ws, L.status));
    double *qbar = reinterpret_cast<double *>(ws_at(ws, L.qbar));
    double *kbar = reinterpret_cast<double *>(ws_at(ws, L.kbar));
    double *kpart = reinterpret_cast<double *>(ws_at(ws, L.kpart));
    double *scores = reinterpret_cast<double *>(ws_at(ws, L.scores));
    int32_t *idx = reinterpret_cast<int32_t *>(ws_at(ws, L.idx));
    uint32_t *amask = reinterpret_cast<uint32_t *>(ws_at(ws, L.amask));
    float *kmean = reinterpret_cast<float *>(ws_at(ws, L.kmean));
    int8_t *q8 = quant ? reinterpret_cast<int8_t *>(ws_at(ws, L.q8)) : nullptr;
    int8_t *k8 = quant ? reinterpret_cast<int8_t *>(ws_at(ws, L.k8)) : nullptr;
    float *qscale = quant ? reinterpret_cast<float *>(ws_at(ws, L.qscale)) : nullptr;
    float *kscale = quant ? reinterpret_cast<float *>(ws_at(ws, L.kscale)) : nullptr;
    uint16_t *states = reinterpret_cast<uint16_t *>(ws_at(ws, L.states));
    float *partials = reinterpret_cast<float *>(ws_at(ws, L.partials));
    float *htot = reinterpret_cast<float *>(ws_at(ws, L.htot));
    float *hq = reinterpret_cast<float *>(ws_at(ws, L.hq));
    uint16_t *v16 = quant ? nullptr : reinterpret_cast<uint16_t *>(ws_at(ws, L.v16));
    int e = 0;
    auto mark = [&]() { if (ev) cudaEventRecord(ev[e++], s); };

    if (reset_status) SLA_TRY(cudaMemsetAsync(status, 0, sizeof(int), s));
    // (not while `s` is being captured into a graph: the second stream is destroyed when the call
    // returns, before the capture ends)
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    SLA_TRY(cudaStreamIsCapturing(s, &cap));
    ForkK fk;
    const bool fork = ev == nullptr && cap == cudaStreamCaptureStatusNone && fk.make();
    if (ev == nullptr && cap == cudaStreamCaptureStatusNone && !fork)
        cudaGetLastError();  // no second stream: run in order on `s`; the failure stays out of the launch checks
    cudaStream_t sk = fork ? fk.st : s;  // the K side's stream
    if (fork) {
        SLA_TRY(cudaEventRecord(fk.ev[0], s));
        SLA_TRY(cudaStreamWaitEvent(sk, fk.ev[0], 0));
    }
    mark();
    // The stages up to the join.  On an error the K side is still joined below, so that nothing
    // this call queued outlives the caller's stream.
    auto until_join = [&]() -> sla_status {
        // (1) Q: INT8 codes and scales, with the pooled block means as a by-product
        //     (without quantisation: the pooled means alone)
        if (quant) SLA_TRY(launch_quant(q, g.BH, N, blk_q, g.n_qb, nullptr, q8, qscale, qbar, quant == 2, s));
        else SLA_TRY(launch_pool(q, g.BH, N, blk_q, g.n_qb, qbar, nullptr, s));
        mark();
        // (2) pooled block means of K (and its partial sums for the smoothing mean),
        //     per-key-block linear states and the global state
        SLA_TRY(launch_pool(k, g.BH, N, blk_k, g.n_kb, kbar, quant ? kpart : nullptr, sk));
        if (fork) SLA_TRY(cudaEventRecord(fk.ev[1], sk));
        SLA_TRY(launch_states(k, v, g, phi, states, partials, v16, status, sk));
        SLA_TRY(launch_htot(partials, g, htot, sk));
        mark();
        // (3) scores + top-k selection
        if (fork) SLA_TRY(cudaStreamWaitEvent(s, fk.ev[1], 0));
        SLA_TRY(launch_scores(qbar, kbar, g, scores, s));
        SLA_TRY(launch_topk(scores, g, idx, nullptr, amask, s));
        mark();
        // (4) K: smoothing mean, INT8 codes and scales
        if (quant) {
            SLA_TRY(launch_kmean(kpart, g.BH, N, pool_parts(g.n_kb), kmean, sk));
            SLA_TRY(launch_quant(k, g.BH, N, blk_k, g.n_kb, kmean, k8, kscale, nullptr, quant == 2, sk));
        }
        return SLA_OK;
    };
    st = until_join();
    if (fork) {  // the join: the state reduction and attention need the K side
        if (cudaEventRecord(fk.ev[2], sk) != cudaSuccess || cudaStreamWaitEvent(s, fk.ev[2], 0) != cudaSuccess) {
            cudaStreamSynchronize(sk);
            return SLA_ERR_CUDA;
        }
    }
    if (st != SLA_OK) return st;
    mark();
    // (5) per-query-block state
    SLA_TRY(launch_state_reduce(amask, states, htot, g, hq, status, s));
    mark();
    // (6) block-sparse attention + linear epilogue + combine
    SLA_TRY(launch_attention(q, k, quant ? v : v16, q8, k8, qscale, kscale, idx, hq, g, phi, out, status, s));
    mark();
    return SLA_OK;
}

// Device memory of sla_forward_host: the workspace of one chunk's forward at offset 0, then two
// staging slots, each holding Q, K, V and the output of one chunk.
struct HostPlan {
    int hc;              // (batch, head) problems per chunk
    size_t ws;           // workspace bytes (a multiple of 256)
    size_t tensor;       // bytes of one staged tensor of a chunk (a multiple of 256)
    size_t total;
};

bool host_plan(int B, int H, int N, int d, int blk_q, int blk_k, float topk, int quant, int chunk_heads, HostPlan &p)
{
    if (check_shape(B, H, N, d, blk_q, blk_k, topk) != SLA_OK || quant < 0 || quant > 2 || chunk_heads < 1)
        return false;
    p.hc = chunk_heads < B * H ? chunk_heads : B * H;
    p.ws = align256(make_layout(make_geometry(1, p.hc, N, d, blk_q, blk_k, topk, quant)).total);
    p.tensor = align256((size_t)p.hc * N * d * sizeof(uint16_t));
    p.total = p.ws + 2 * 4 * p.tensor;
    return true;
}

// Streams and events of one sla_forward_host call; released when the call returns (CUDA frees
// them once the work queued on them has completed).
struct HostPipe {
    cudaStream_t st[3] = {nullptr, nullptr, nullptr};  // copy-in, compute, copy-out
    std::vector<cudaEvent_t> ev;
    ~HostPipe()
    {
        for (cudaEvent_t e : ev) cudaEventDestroy(e);
        for (cudaStream_t x : st)
            if (x) cudaStreamDestroy(x);
    }
    bool make(int n_events)
    {
        for (cudaStream_t &x : st)
            if (cudaStreamCreateWithFlags(&x, cudaStreamNonBlocking) != cudaSuccess) return false;
        ev.reserve(n_events);
        for (int i = 0; i < n_events; ++i) {
            cudaEvent_t e;
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
            ev.push_back(e);
        }
        return true;
    }
};

}  // namespace

extern "C" {

size_t sla_forward_host_bytes(int B, int H, int N, int d, int blk_q, int blk_k, float topk, int quant,
                              int chunk_heads)
{
    HostPlan p;
    return host_plan(B, H, N, d, blk_q, blk_k, topk, quant, chunk_heads, p) ? p.total : 0;
}

sla_status sla_forward_host(const void *q_host, const void *k_host, const void *v_host, void *out_host, int B, int H,
                            int N, int d, int blk_q, int blk_k, float topk, int phi, int quant, int chunk_heads,
                            void *dev, size_t dev_bytes, void *stream)
{
    sla_status st = check_shape(B, H, N, d, blk_q, blk_k, topk);
    if (st != SLA_OK) return st;
    if (phi != SLA_PHI_ELU1 && phi != SLA_PHI_RELU) return SLA_ERR_INVALID_ARG;
    if (quant < 0 || quant > 2 || chunk_heads < 1) return SLA_ERR_INVALID_ARG;
    if (!q_host || !k_host || !v_host || !out_host || !aligned16(dev)) return SLA_ERR_INVALID_ARG;
    HostPlan p;
    if (!host_plan(B, H, N, d, blk_q, blk_k, topk, quant, chunk_heads, p)) return SLA_ERR_INVALID_ARG;
    if (dev_bytes < p.total) return SLA_ERR_WORKSPACE;

    const int BH = B * H, n_chunks = (BH + p.hc - 1) / p.hc;
    const size_t head_bytes = (size_t)N * d * sizeof(uint16_t);
    char *base = static_cast<char *>(dev);
    void *ws = base;  // status word at offset 0: sla_check(dev, stream) reads the call's status
    auto staged = [&](int c, int t) { return base + p.ws + ((size_t)(c & 1) * 4 + t) * p.tensor; };
    const char *host_in[3] = {static_cast<const char *>(q_host), static_cast<const char *>(k_host),
                              static_cast<const char *>(v_host)};
    char *host_out = static_cast<char *>(out_host);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // events: [0] the caller's stream at entry; per chunk c: inputs landed (1 + 3c), forward done
    // (2 + 3c), output copied out (3 + 3c)
    HostPipe pipe;
    if (!pipe.make(1 + 3 * n_chunks)) {
        cudaGetLastError();  // reported here; later calls' launch checks do not see it
        return SLA_ERR_CUDA;
    }
    cudaStream_t s_in = pipe.st[0], s_cmp = pipe.st[1], s_out = pipe.st[2];
    auto ev_in = [&](int c) { return pipe.ev[1 + 3 * c]; };
    auto ev_done = [&](int c) { return pipe.ev[2 + 3 * c]; };
    auto ev_out = [&](int c) { return pipe.ev[3 + 3 * c]; };
    SLA_TRY(cudaEventRecord(pipe.ev[0], s));
    for (cudaStream_t x : pipe.st) SLA_TRY(cudaStreamWaitEvent(x, pipe.ev[0], 0));

    // Chunk c uses slot c % 2.  Its copy-in waits for the forward of chunk c - 2 (which read the
    // slot's inputs), its forward for its copy-in and for the copy-out of chunk c - 2 (which read
    // the slot's output).  Every event is recorded before a wait on it is queued.
    auto enqueue = [&]() -> sla_status {
        for (int c = 0; c < n_chunks; ++c) {
            const int h0 = c * p.hc, nh = (c + 1) * p.hc <= BH ? p.hc : BH - h0;
            const size_t off = (size_t)h0 * head_bytes, bytes = (size_t)nh * head_bytes;
            if (c >= 2) SLA_TRY(cudaStreamWaitEvent(s_in, ev_done(c - 2), 0));
            for (int t = 0; t < 3; ++t)
                SLA_TRY(cudaMemcpyAsync(staged(c, t), host_in[t] + off, bytes, cudaMemcpyHostToDevice, s_in));
            SLA_TRY(cudaEventRecord(ev_in(c), s_in));

            SLA_TRY(cudaStreamWaitEvent(s_cmp, ev_in(c), 0));
            if (c >= 2) SLA_TRY(cudaStreamWaitEvent(s_cmp, ev_out(c - 2), 0));
            // the first chunk clears the status word; later chunks keep an error recorded before them
            st = run_forward(staged(c, 0), staged(c, 1), staged(c, 2), staged(c, 3), 1, nh, N, d, blk_q, blk_k, topk,
                             phi, quant, ws, p.ws, s_cmp, nullptr, c == 0);
            if (st != SLA_OK) return st;
            SLA_TRY(cudaEventRecord(ev_done(c), s_cmp));

            SLA_TRY(cudaStreamWaitEvent(s_out, ev_done(c), 0));
            SLA_TRY(cudaMemcpyAsync(host_out + off, staged(c, 3), bytes, cudaMemcpyDeviceToHost, s_out));
            SLA_TRY(cudaEventRecord(ev_out(c), s_out));
        }
        // the caller's stream continues after the last copy-out (which follows every other step)
        SLA_TRY(cudaStreamWaitEvent(s, ev_out(n_chunks - 1), 0));
        return SLA_OK;
    };
    st = enqueue();
    if (st != SLA_OK)  // nothing queued by this call outlives it
        for (cudaStream_t x : pipe.st) cudaStreamSynchronize(x);
    return st;
}

sla_status sla_forward(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d, int blk_q,
                       int blk_k, float topk, int phi, int quant, void *ws, size_t ws_bytes, void *stream)
{
    return run_forward(q, k, v, out, B, H, N, d, blk_q, blk_k, topk, phi, quant, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream), nullptr);
}

size_t sla_backward_workspace_bytes(int B, int H, int N, int d, int blk_q, int blk_k, float topk)
{
    if (check_shape(B, H, N, d, blk_q, blk_k, topk) != SLA_OK) return 0;
    return backward_workspace_bytes(make_geometry(B, H, N, d, blk_q, blk_k, topk, 0));
}

sla_status sla_backward(const void *q, const void *k, const void *v, const void *dout, float *dq, float *dk, float *dv,
                        int B, int H, int N, int d, int blk_q, int blk_k, float topk, int phi, void *ws,
                        size_t ws_bytes, void *stream)
{
    sla_status st = check_shape(B, H, N, d, blk_q, blk_k, topk);
    if (st != SLA_OK) return st;
    if (phi != SLA_PHI_ELU1 && phi != SLA_PHI_RELU) return SLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
        !aligned16(dv) || !aligned16(ws))
        return SLA_ERR_INVALID_ARG;
    const Geometry g = make_geometry(B, H, N, d, blk_q, blk_k, topk, 0);
    if (ws_bytes < backward_workspace_bytes(g)) return SLA_ERR_WORKSPACE;
    SLA_TRY(launch_backward(q, k, v, dout, dq, dk, dv, g, phi, ws, static_cast<cudaStream_t>(stream)));
    return SLA_OK;
}

sla_status sla_forward_profile(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d,
                               int blk_q, int blk_k, float topk, int phi, int quant, void *ws, size_t ws_bytes,
                               void *stream, float *stage_ms)
{
    if (!stage_ms) return SLA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaEvent_t ev[kProfStages];
    int made = 0;
    for (; made < kProfStages; ++made)
        if (cudaEventCreate(&ev[made]) != cudaSuccess) break;
    sla_status st = made == kProfStages ? SLA_OK : SLA_ERR_CUDA;
    if (st == SLA_OK) st = run_forward(q, k, v, out, B, H, N, d, blk_q, blk_k, topk, phi, quant, ws, ws_bytes, s, ev);
    if (st == SLA_OK && cudaEventSynchronize(ev[kProfStages - 1]) != cudaSuccess) st = SLA_ERR_CUDA;
    if (st == SLA_OK) {
        for (int i = 0; i + 1 < kProfStages; ++i)
            if (cudaEventElapsedTime(&stage_ms[i], ev[i], ev[i + 1]) != cudaSuccess) st = SLA_ERR_CUDA;
        if (cudaEventElapsedTime(&stage_ms[kProfStages - 1], ev[0], ev[kProfStages - 1]) != cudaSuccess)
            st = SLA_ERR_CUDA;
    }
    for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
    return st;
}

sla_status sla_set_wait_budget(long long cycles)
{
    if (cycles < 0) return SLA_ERR_INVALID_ARG;
    if (set_wait_budget_attention(cycles) != cudaSuccess || set_wait_budget_linear(cycles) != cudaSuccess ||
        set_wait_budget_w8a8(cycles) != cudaSuccess || set_wait_budget_bwd(cycles) != cudaSuccess)
        return SLA_ERR_CUDA;
    return SLA_OK;
}

sla_status sla_check(void *ws, void *stream)
{
    if (!aligned16(ws)) return SLA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return SLA_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SLA_ERR_CUDA;
    return h == 0 ? SLA_OK : (sla_status)h;
}

}  // extern "C"
