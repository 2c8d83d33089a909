// moe_api.cu -- the extern "C" entry points of libmoe.so (declared in include/moe.h).
//
// Host side only: argument validation (every error is returned before anything is enqueued),
// the workspace layout, and the choice of kernels.  All arithmetic of the layer runs in the
// kernels of k_route.cu, k_ffn.cu and k_gemm_tc.cu.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <vector>

#include "moe_internal.cuh"

struct moe_arena {
    const uint8_t *base;
    size_t bytes;
    int H, F, E, shared;      // shared: index of the shared expert (== E) or -1
    int n;                    // descriptors (E or E + 1)
    int fmt_mask;             // bit f set when some expert uses format f
    int max_stride01, max_stride2;
    moe::ExpertDev *d_experts;
    void *d_wmaps;            // tensor maps of the packed matrices (tensor-core path) or null
    bool tc_ok;               // large batches may run on the tensor cores
    cudaEvent_t ev[3];        // optional timing events around the tensor-core phases
    uint64_t wait_ns;         // limit of every bounded wait inside the kernels
    std::vector<moe_expert_desc> descs;
};

namespace moe {

static std::atomic<unsigned long long> g_kernels{0};

void note_launches(int n) { g_kernels.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

cudaError_t ensure_smem_impl(const void *kernel, size_t bytes) {
    static std::mutex mu;
    static std::map<std::pair<int, const void *>, size_t> done;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(mu);
    size_t &have = done[{dev, kernel}];
    if (bytes <= have) return cudaSuccess;
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (err == cudaSuccess) have = bytes;
    return err;
}

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

static bool aligned(const void *p, size_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

WsLayout ws_layout(const moe_arena *A, int T, int k, uint32_t flags, bool allow_tc) {
    WsLayout L{};
    size_t p = 0;
    auto take = [&](size_t bytes) {
        const size_t o = p;
        p = align256(p + bytes);
        return o;
    };
    const int H = A->H, F = A->F, E = A->E;
    const int shared = A->shared >= 0 ? 1 : 0;
    L.slots = T * k + T;
    L.hpad = ((F + 255) / 256) * 256;
    L.max_jobs = std::min(E, T * k) + shared;
    L.n_chunks = (T + kChunk - 1) / kChunk;
    L.status = take(sizeof(uint32_t));
    L.sync = take(4 * sizeof(uint32_t));                                  // fused-decode counters
    L.blkcnt = take(sizeof(uint32_t) * (size_t)L.max_jobs * (F / 32));    // rows done per h block
    L.njobs = take(sizeof(int32_t));
    L.jobs = take(sizeof(Job) * (size_t)L.max_jobs);
    L.xq = take((size_t)T * H);
    L.xd = take((size_t)T * (H / 32) * 2);
    L.xs = take((size_t)T * (H / 32) * 2);
    L.xsum = take((size_t)T * (H / 32) * 4);
    L.ids = take((size_t)T * k * 4);
    L.w = take((size_t)T * k * 4);
    L.counts = take((size_t)E * 4);
    L.offsets = take((size_t)(E + 1) * 4);
    L.perm = take((size_t)T * k * 4);
    L.inv_perm = take((size_t)T * k * 4);
    L.chunk_counts = take((size_t)L.n_chunks * E * 4);
    L.chunk_base = take((size_t)L.n_chunks * E * 4);
    L.hq = take((size_t)L.slots * L.hpad);
    L.hd = take((size_t)L.slots * (L.hpad / 32) * 2);
    L.hs = take((size_t)L.slots * (L.hpad / 32) * 2);
    L.hsum = take((size_t)L.slots * (L.hpad / 32) * 4);
    L.h = take((size_t)L.slots * F * 4);
    (void)flags;
    L.y = (flags & MOE_F_DETERMINISTIC) ? take((size_t)L.slots * H * 4) : 0;
    // the tensor-core operands come last
    L.tc = allow_tc && A->tc_ok && ((flags & MOE_F_FORCE_PREFILL) || T > kDecodeMaxT) &&
           !(flags & MOE_F_FORCE_DECODE);
    L.kd = ((F + 63) / 64) * 64;
    if (L.tc) {
        L.xh = take((size_t)T * H * 2);
        L.xl = take((size_t)T * H * 2);
        L.xsh = take((size_t)T * (H / 32) * 4);
        L.xsl = take((size_t)T * (H / 32) * 4);
        L.xscale = take((size_t)T * 4);
        L.hh = take((size_t)L.slots * L.kd * 2);
        L.hscale = take((size_t)L.slots * 4);
    }
    L.total = p;
    return L;
}

moe_status check_forward_args(const moe_arena *arena, const float *d_x, const float *d_logits,
                              int T, int k, const float *d_out, uint32_t flags) {
    if (!arena || !d_x || !d_logits || !d_out) return MOE_ERR_INVALID_ARG;
    if (T <= 0 || k <= 0 || k > kMaxK || k > arena->E) return MOE_ERR_INVALID_ARG;
    if ((flags & MOE_F_FORCE_DECODE) && (flags & MOE_F_FORCE_PREFILL)) return MOE_ERR_INVALID_ARG;
    if (!aligned(d_x, 16) || !aligned(d_out, 16) || !aligned(d_logits, 4)) return MOE_ERR_ALIGNMENT;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

uint64_t moe_kernels_enqueued(void) { return (uint64_t)g_kernels.load(); }

const char *moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or format";
        case MOE_ERR_ALIGNMENT: return "misaligned pointer or stride";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_NONFINITE: return "non-finite input";
        case MOE_ERR_BOUNDS: return "descriptor outside the arena";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
        case MOE_ERR_WORKSPACE: return "workspace too small";
    }
    return "unknown status";
}

moe_status moe_arena_create(const void *d_arena, size_t arena_bytes, int hidden, int ffn,
                            int n_experts, int shared_expert, const moe_expert_desc *host_descs,
                            moe_arena **out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!d_arena || !host_descs || hidden <= 0 || ffn <= 0 || n_experts <= 0) return MOE_ERR_INVALID_ARG;
    if (hidden % 32 || ffn % 32) return MOE_ERR_INVALID_ARG;
    if (n_experts > kMaxE) return MOE_ERR_UNSUPPORTED;
    if (hidden > 4096 || ffn > 4096) return MOE_ERR_UNSUPPORTED;
    if (shared_expert != -1 && shared_expert != n_experts) return MOE_ERR_INVALID_ARG;
    if (!aligned(d_arena, 256)) return MOE_ERR_ALIGNMENT;
    const int n = n_experts + (shared_expert >= 0 ? 1 : 0);
    std::vector<ExpertDev> dev(n);
    int fmt_mask = 0;
    uint64_t ms01 = 0, ms2 = 0;
    for (int e = 0; e < n; e++) {
        const moe_expert_desc &d = host_descs[e];
        if (d.fmt < 0 || d.fmt > MOE_FMT_Q6_K || d.reserved != 0) return MOE_ERR_INVALID_ARG;
        const int bw = block_weights(d.fmt), bb = block_bytes(d.fmt);
        if (hidden % bw) return MOE_ERR_UNSUPPORTED;
        const int rows[3] = {ffn, ffn, hidden};
        const int width[3] = {hidden, hidden, ffn};
        for (int t = 0; t < 3; t++) {
            const uint64_t packed = (uint64_t)((width[t] + bw - 1) / bw) * bb;
            if (d.off[t] % 16 || d.stride[t] % 16) return MOE_ERR_ALIGNMENT;
            if (d.stride[t] < packed || d.stride[t] > (1u << 30)) return MOE_ERR_INVALID_ARG;
            const uint64_t end = d.off[t] + (uint64_t)(rows[t] - 1) * d.stride[t] + packed;
            if (d.off[t] > arena_bytes || end > arena_bytes) return MOE_ERR_BOUNDS;
            dev[e].m[t] = static_cast<const uint8_t *>(d_arena) + d.off[t];
            dev[e].stride[t] = (uint32_t)d.stride[t];
        }
        dev[e].fmt = d.fmt;
        dev[e].pad = 0;
        ms01 = std::max(ms01, std::max(d.stride[0], d.stride[1]));
        ms2 = std::max(ms2, d.stride[2]);
        fmt_mask |= 1 << d.fmt;
    }
    moe_arena *A = new (std::nothrow) moe_arena();
    if (!A) return MOE_ERR_CUDA;
    A->base = static_cast<const uint8_t *>(d_arena);
    A->bytes = arena_bytes;
    A->H = hidden;
    A->F = ffn;
    A->E = n_experts;
    A->shared = shared_expert;
    A->n = n;
    A->fmt_mask = fmt_mask;
    A->max_stride01 = (int)ms01;
    A->max_stride2 = (int)ms2;
    A->descs.assign(host_descs, host_descs + n);
    A->d_wmaps = nullptr;
    A->tc_ok = false;
    A->ev[0] = A->ev[1] = A->ev[2] = nullptr;
    A->wait_ns = 2000000000ull;
    if (cudaMalloc(&A->d_experts, sizeof(ExpertDev) * n) != cudaSuccess ||
        cudaMemcpy(A->d_experts, dev.data(), sizeof(ExpertDev) * n, cudaMemcpyHostToDevice) !=
            cudaSuccess) {
        cudaFree(A->d_experts);
        delete A;
        return MOE_ERR_CUDA;
    }
    // tensor-core path: weight tensor maps, and a shared-memory plan that fits this device
    {
        std::vector<uint8_t> maps;
        int dev_id = 0, optin = 0;
        const bool fits = cudaGetDevice(&dev_id) == cudaSuccess &&
                          cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                                 dev_id) == cudaSuccess &&
                          !(fmt_mask & (1 << MOE_FMT_Q6_K)) &&
                          tc_smem_bytes(fmt_mask) <= (size_t)optin && ffn % 64 == 0;
        if (fits && tc_build_weight_maps(A->base, host_descs, n, hidden, ffn, maps)) {
            if (cudaMalloc(&A->d_wmaps, maps.size()) != cudaSuccess ||
                cudaMemcpy(A->d_wmaps, maps.data(), maps.size(), cudaMemcpyHostToDevice) !=
                    cudaSuccess) {
                cudaFree(A->d_wmaps);
                cudaFree(A->d_experts);
                delete A;
                return MOE_ERR_CUDA;
            }
            A->tc_ok = true;
        }
    }
    *out = A;
    return MOE_OK;
}

void moe_arena_destroy(moe_arena *arena) {
    if (!arena) return;
    cudaFree(arena->d_experts);
    cudaFree(arena->d_wmaps);
    delete arena;
}

moe_status moe_workspace_size(const moe_arena *arena, int max_tokens, int k, uint32_t flags,
                              size_t *bytes) {
    if (!arena || !bytes || max_tokens <= 0 || k <= 0 || k > kMaxK || k > arena->E)
        return MOE_ERR_INVALID_ARG;
    *bytes = ws_layout(arena, max_tokens, k, flags).total;
    return MOE_OK;
}

moe_status moe_quantize_act(const float *d_x, int T, int H, int8_t *d_q, uint16_t *d_d,
                            uint16_t *d_s, uint32_t *d_status, void *stream) {
    if (!d_x || !d_q || !d_d || !d_s || T < 0 || H <= 0 || H % 32) return MOE_ERR_INVALID_ARG;
    if (!aligned(d_x, 16) || !aligned(d_q, 16) || !aligned(d_d, 2) || !aligned(d_s, 2))
        return MOE_ERR_ALIGNMENT;
    if (launch_quantize(d_x, (int64_t)T * H / 32, d_q, d_d, d_s, nullptr, d_status,
                        (cudaStream_t)stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

static size_t route_ws_bytes(int T, int E, int k) {
    const int n_chunks = (T + kChunk - 1) / kChunk;
    size_t p = 0;
    p = align256(p + (size_t)n_chunks * E * 4);   // chunk counts
    p = align256(p + (size_t)n_chunks * E * 4);   // chunk cursors
    p = align256(p + sizeof(Job) * (size_t)(std::min(E, T * k) + 1));
    p = align256(p + 4);
    return p;
}

moe_status moe_route_workspace_size(int T, int E, int k, size_t *bytes) {
    if (!bytes || T <= 0 || E <= 0 || k <= 0 || k > kMaxK || k > E) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE) return MOE_ERR_UNSUPPORTED;
    *bytes = route_ws_bytes(T, E, k);
    return MOE_OK;
}

moe_status moe_route_topk(const float *d_logits, int T, int E, int k, int32_t *d_ids,
                          float *d_w, int32_t *d_counts, int32_t *d_offsets, int32_t *d_perm,
                          int32_t *d_inv_perm, uint32_t *d_status, void *d_ws, size_t ws_bytes,
                          void *stream) {
    if (!d_logits || !d_ids || !d_w || !d_counts || !d_offsets || !d_perm || !d_ws)
        return MOE_ERR_INVALID_ARG;
    if (T <= 0 || E <= 0 || k <= 0 || k > kMaxK || k > E) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE) return MOE_ERR_UNSUPPORTED;
    if (!aligned(d_ws, 256)) return MOE_ERR_ALIGNMENT;
    if (ws_bytes < route_ws_bytes(T, E, k)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    const int n_chunks = (T + kChunk - 1) / kChunk;
    uint8_t *ws = static_cast<uint8_t *>(d_ws);
    int32_t *cc = reinterpret_cast<int32_t *>(ws);
    int32_t *cb = reinterpret_cast<int32_t *>(ws + align256((size_t)n_chunks * E * 4));
    Job *jobs = reinterpret_cast<Job *>(ws + 2 * align256((size_t)n_chunks * E * 4));
    int32_t *nj = reinterpret_cast<int32_t *>(
        ws + 2 * align256((size_t)n_chunks * E * 4) +
        align256(sizeof(Job) * (size_t)(std::min(E, T * k) + 1)));
    if (launch_topk(d_logits, T, E, k, d_ids, d_w, d_status, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (launch_group(d_ids, T, k, E, 0, d_counts, d_offsets, d_perm, d_inv_perm, cc, cb, jobs, nj,
                     st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status moe_ws_views(const moe_arena *arena, void *d_ws, int T, int k, uint32_t flags,
                        moe_ws_view *out) {
    if (!arena || !d_ws || !out || T <= 0 || k <= 0 || k > kMaxK || k > arena->E)
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(arena, T, k, flags);
    uint8_t *ws = static_cast<uint8_t *>(d_ws);
    out->status = reinterpret_cast<uint32_t *>(ws + L.status);
    out->xq = reinterpret_cast<int8_t *>(ws + L.xq);
    out->xd = reinterpret_cast<uint16_t *>(ws + L.xd);
    out->xs = reinterpret_cast<uint16_t *>(ws + L.xs);
    out->ids = reinterpret_cast<int32_t *>(ws + L.ids);
    out->w = reinterpret_cast<float *>(ws + L.w);
    out->counts = reinterpret_cast<int32_t *>(ws + L.counts);
    out->offsets = reinterpret_cast<int32_t *>(ws + L.offsets);
    out->perm = reinterpret_cast<int32_t *>(ws + L.perm);
    out->inv_perm = reinterpret_cast<int32_t *>(ws + L.inv_perm);
    out->hq = reinterpret_cast<int8_t *>(ws + L.hq);
    out->hd = reinterpret_cast<uint16_t *>(ws + L.hd);
    out->hs = reinterpret_cast<uint16_t *>(ws + L.hs);
    out->h = (flags & MOE_F_KEEP_H) ? reinterpret_cast<float *>(ws + L.h) : nullptr;
    out->slots = L.slots;
    out->hpad = L.hpad;
    out->counters = reinterpret_cast<uint32_t *>(ws + L.sync);
    return MOE_OK;
}

moe_status moe_read_status(uint32_t *d_status_word, void *stream, int clear,
                           moe_status *device_status) {
    if (!d_status_word || !device_status) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, d_status_word, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (clear && cudaMemsetAsync(d_status_word, 0, 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    *device_status = (moe_status)v;
    return MOE_OK;
}

}  // extern "C"

namespace moe {

// Every host-side check of moe_forward, in its order.
static moe_status forward_checks(const moe_arena *arena, const float *d_x, const float *d_logits,
                                 int T, int k, const float *d_out, const void *d_ws,
                                 size_t ws_bytes, uint32_t flags) {
    const moe_status chk = check_forward_args(arena, d_x, d_logits, T, k, d_out, flags);
    if (chk != MOE_OK) return chk;
    if (!d_ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(d_ws, 256)) return MOE_ERR_ALIGNMENT;
    if ((flags & MOE_F_FORCE_PREFILL) && !arena->tc_ok) return MOE_ERR_UNSUPPORTED;
    if (ws_bytes < ws_layout(arena, T, k, flags).total) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

// moe_forward with an optional per-token weight of the shared expert's output (d_gate [T]) and
// an optional router lookahead for the next layer of a chain, which the decode kernel runs
// inside when it can (*look_fused; otherwise the caller runs it).
static moe_status forward_impl(const moe_arena *arena, const float *d_x, const float *d_logits,
                               const float *d_gate, int T, int k, float *d_out, void *d_ws,
                               size_t ws_bytes, uint32_t flags, void *stream,
                               const Lookahead *look = nullptr, bool *look_fused = nullptr) {
    if (look_fused) *look_fused = false;
    const moe_status chk = forward_checks(arena, d_x, d_logits, T, k, d_out, d_ws, ws_bytes, flags);
    if (chk != MOE_OK) return chk;
    const WsLayout L = ws_layout(arena, T, k, flags);
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *ws = static_cast<uint8_t *>(d_ws);
    const int H = arena->H, E = arena->E;
    const int shared = arena->shared >= 0 ? 1 : 0;
    const bool decode = (flags & MOE_F_FORCE_DECODE) ||
                        (!(flags & MOE_F_FORCE_PREFILL) && T <= kDecodeMaxT);

    uint32_t *status = reinterpret_cast<uint32_t *>(ws + L.status);
    int8_t *xq = reinterpret_cast<int8_t *>(ws + L.xq);
    uint16_t *xd = reinterpret_cast<uint16_t *>(ws + L.xd);
    uint16_t *xs = reinterpret_cast<uint16_t *>(ws + L.xs);
    float *xsum = reinterpret_cast<float *>(ws + L.xsum);
    int32_t *ids = reinterpret_cast<int32_t *>(ws + L.ids);
    float *w = reinterpret_cast<float *>(ws + L.w);
    int32_t *counts = reinterpret_cast<int32_t *>(ws + L.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(ws + L.offsets);
    int32_t *perm = reinterpret_cast<int32_t *>(ws + L.perm);
    int32_t *inv_perm = reinterpret_cast<int32_t *>(ws + L.inv_perm);
    Job *jobs = reinterpret_cast<Job *>(ws + L.jobs);
    int32_t *njobs = reinterpret_cast<int32_t *>(ws + L.njobs);

    if (decode && T <= kDecodeMaxT) {
        FfnArgs a{};
        a.experts = arena->d_experts;
        a.out = d_out;
        a.status = status;
        a.T = T;
        a.k = k;
        a.H = H;
        a.F = arena->F;
        a.hpad = L.hpad;
        a.max_jobs = L.max_jobs;
        a.fmt_mask = arena->fmt_mask;
        a.max_stride01 = arena->max_stride01;
        a.max_stride2 = arena->max_stride2;
        a.h = (flags & MOE_F_KEEP_H) ? reinterpret_cast<float *>(ws + L.h) : nullptr;
        a.gate = d_gate;
        a.wait_ns = arena->wait_ns;
        if (look) a.look = *look;
        bool taken = false, fused = false;
        cudaError_t e = launch_decode_fused(a, E, shared, d_x, d_logits, ws, L, L.sync, L.blkcnt,
                                            true, st, &taken, &fused);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        if (look_fused) *look_fused = fused;
        if (taken) return MOE_OK;
    }
    // a1-a3
    const bool small_route = T <= kDecodeMaxT && T * k <= kDecodeMaxT * kMaxK &&
                             ((size_t)T * E + E) * 4 <= 96 * 1024;
    const bool tc = L.tc && !(decode && T <= kDecodeMaxT);
    cudaError_t err;
    if (small_route && !tc) {
        err = launch_route_small(d_x, d_logits, T, H, E, k, shared, L, ws, st);
    } else {
        if (tc && !(flags & MOE_F_TC_I8))   // the kind::f16 operand planes as well
            err = launch_quant_rows(d_x, T, H, xq, xd, xs, xsum,
                                    reinterpret_cast<__half *>(ws + L.xh),
                                    reinterpret_cast<__half *>(ws + L.xl),
                                    reinterpret_cast<float *>(ws + L.xsh),
                                    reinterpret_cast<float *>(ws + L.xsl),
                                    reinterpret_cast<float *>(ws + L.xscale), status, st);
        else
            err = launch_quantize(d_x, (int64_t)T * H / 32, xq, xd, xs, xsum, status, st);
        if (err == cudaSuccess) err = launch_topk(d_logits, T, E, k, ids, w, status, st);
        if (err == cudaSuccess)
            err = launch_group(ids, T, k, E, shared, counts, offsets, perm, inv_perm,
                               reinterpret_cast<int32_t *>(ws + L.chunk_counts),
                               reinterpret_cast<int32_t *>(ws + L.chunk_base), jobs, njobs, st);
    }
    if (err != cudaSuccess) {
        if (std::getenv("MOE_DEBUG"))
            std::fprintf(stderr, "moe: routing failed: %s\n", cudaGetErrorString(err));
        return MOE_ERR_CUDA;
    }

    FfnArgs a{};
    a.experts = arena->d_experts;
    a.jobs = jobs;
    a.njobs = njobs;
    a.perm = perm;
    a.inv_perm = inv_perm;
    a.w = w;
    a.xq = xq;
    a.xd = xd;
    a.xsum = xsum;
    a.hq = reinterpret_cast<int8_t *>(ws + L.hq);
    a.hd = reinterpret_cast<uint16_t *>(ws + L.hd);
    a.hs = reinterpret_cast<uint16_t *>(ws + L.hs);
    a.hsum = reinterpret_cast<float *>(ws + L.hsum);
    a.h = reinterpret_cast<float *>(ws + L.h);
    a.y = (flags & MOE_F_DETERMINISTIC) ? reinterpret_cast<float *>(ws + L.y) : nullptr;
    a.out = d_out;
    a.gate = d_gate;
    a.status = status;
    a.T = T;
    a.k = k;
    a.H = H;
    a.F = arena->F;
    a.hpad = L.hpad;
    a.max_jobs = L.max_jobs;
    a.fmt_mask = arena->fmt_mask;
    a.max_stride01 = arena->max_stride01;
    a.max_stride2 = arena->max_stride2;
    a.wait_ns = arena->wait_ns;

    if (tc) {
        // a4-a7 on the tensor cores
        TcPhaseArgs p{};
        p.ffn = a;
        p.wmaps = arena->d_wmaps;
        p.slots = L.slots;
        p.keep_h = (flags & MOE_F_KEEP_H) ? 1 : 0;
        p.i8 = (flags & MOE_F_TC_I8) ? 1 : 0;
        p.Kd = L.kd;
        p.xh = reinterpret_cast<const __half *>(ws + L.xh);
        p.xl = reinterpret_cast<const __half *>(ws + L.xl);
        p.xsh = reinterpret_cast<const float *>(ws + L.xsh);
        p.xsl = reinterpret_cast<const float *>(ws + L.xsl);
        p.xscale = reinterpret_cast<const float *>(ws + L.xscale);
        p.hh = reinterpret_cast<const __half *>(ws + L.hh);
        p.hscale = reinterpret_cast<const float *>(ws + L.hscale);
        p.wait_ns = arena->wait_ns;
        const int used = T * k + (shared ? T : 0);
        if (p.keep_h) err = launch_hpad_zero(a, st);
        if (err == cudaSuccess && !(flags & MOE_F_DETERMINISTIC))
            err = cudaMemsetAsync(d_out, 0, (size_t)T * H * sizeof(float), st);
        if (err == cudaSuccess && arena->ev[0]) err = cudaEventRecord(arena->ev[0], st);
        if (err == cudaSuccess) {
            p.phase = 0;
            err = launch_gemm_tc(p, st);
        }
        if (err == cudaSuccess && arena->ev[1]) err = cudaEventRecord(arena->ev[1], st);
        if (err == cudaSuccess)
            err = launch_h_rows(a.hq, a.hd, used, arena->F, L.hpad, L.kd,
                                reinterpret_cast<__half *>(ws + L.hh),
                                reinterpret_cast<float *>(ws + L.hscale), st);
        if (err == cudaSuccess) {
            p.phase = 1;
            err = launch_gemm_tc(p, st);
        }
        if (err == cudaSuccess && arena->ev[2]) err = cudaEventRecord(arena->ev[2], st);
        if (err == cudaSuccess && (flags & MOE_F_DETERMINISTIC))
            err = launch_combine(a, shared != 0, st);
        if (err != cudaSuccess && std::getenv("MOE_DEBUG"))
            std::fprintf(stderr, "moe: tensor-core path failed: %s\n", cudaGetErrorString(err));
        return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    }
    // a4 + a5
    err = launch_gateup_gemv(a, st);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    // a6 + a7
    if (decode && T <= kDecodeMaxT) {
        err = launch_down_decode(a, st);
    } else if (flags & MOE_F_DETERMINISTIC) {
        err = launch_down_grouped(a, true, st);
        if (err == cudaSuccess) err = launch_combine(a, shared != 0, st);
    } else {
        err = cudaMemsetAsync(d_out, 0, (size_t)T * H * sizeof(float), st);
        if (err == cudaSuccess) err = launch_down_grouped(a, false, st);
    }
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe

extern "C" {

moe_status moe_forward(const moe_arena *arena, const float *d_x, const float *d_logits, int T,
                       int k, float *d_out, void *d_ws, size_t ws_bytes, uint32_t flags,
                       void *stream) {
    return forward_impl(arena, d_x, d_logits, nullptr, T, k, d_out, d_ws, ws_bytes,
                        flags & ~MOE_F_LOOKAHEAD, stream);
}

moe_status moe_set_timing_events(moe_arena *arena, void *ev_begin, void *ev_mid, void *ev_end) {
    if (!arena) return MOE_ERR_INVALID_ARG;
    if ((ev_begin == nullptr) != (ev_mid == nullptr) || (ev_mid == nullptr) != (ev_end == nullptr))
        return MOE_ERR_INVALID_ARG;
    arena->ev[0] = static_cast<cudaEvent_t>(ev_begin);
    arena->ev[1] = static_cast<cudaEvent_t>(ev_mid);
    arena->ev[2] = static_cast<cudaEvent_t>(ev_end);
    return MOE_OK;
}

moe_status moe_set_wait_limit(moe_arena *arena, uint64_t ns) {
    if (!arena || ns == 0) return MOE_ERR_INVALID_ARG;
    arena->wait_ns = ns;
    return MOE_OK;
}

moe_status moe_debug_dequant(const moe_arena *arena, int expert, int which, float *d_out,
                             void *stream) {
    if (!arena || !d_out || expert < 0 || expert >= arena->n || which < 0 || which > 2)
        return MOE_ERR_INVALID_ARG;
    const moe_expert_desc &d = arena->descs[expert];
    const int bw = block_weights(d.fmt);
    const int rows = which < 2 ? arena->F : arena->H;
    const int width = which < 2 ? arena->H : arena->F;
    const int nb = (width + bw - 1) / bw;
    if (launch_dequant(arena->base + d.off[which], d.fmt, rows, nb, (int)d.stride[which], d_out,
                       (cudaStream_t)stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ router in front, chains

namespace moe {

// Host checks of one layer's router and gate rows.
static moe_status check_router_rows(const moe_arena *arena, const float *d_router,
                                    const float *d_gate_row) {
    if (!d_router) return MOE_ERR_INVALID_ARG;
    if (d_gate_row && arena->shared < 0) return MOE_ERR_INVALID_ARG;
    if (arena->H % 4) return MOE_ERR_INVALID_ARG;
    if (!aligned(d_router, 16) || (d_gate_row && !aligned(d_gate_row, 16))) return MOE_ERR_ALIGNMENT;
    return MOE_OK;
}

// A chain workspace: the largest layer workspace, then the chain's own buffers.
struct ChainLayout {
    size_t fwd, xa, xb, xn, out, logits, next, gate, pred, total;
    int H, Emax;
};

static moe_status chain_layout(const moe_chain_layer *ls, int n, int T, int k, uint32_t flags,
                               ChainLayout &C) {
    if (!ls || n <= 0 || T <= 0 || k <= 0 || k > kMaxK) return MOE_ERR_INVALID_ARG;
    if ((flags & MOE_F_LOOKAHEAD) && T > kDecodeMaxT) return MOE_ERR_INVALID_ARG;
    if ((T + 15) / 16 > 65535) return MOE_ERR_UNSUPPORTED;
    C = ChainLayout{};
    const uint32_t ff = flags & ~MOE_F_LOOKAHEAD;
    for (int l = 0; l < n; l++) {
        const moe_arena *A = ls[l].arena;
        if (!A || k > A->E) return MOE_ERR_INVALID_ARG;
        if (l == 0) C.H = A->H;
        if (A->H != C.H) return MOE_ERR_INVALID_ARG;
        const moe_status r = check_router_rows(A, ls[l].d_router, ls[l].d_gate_row);
        if (r != MOE_OK) return r;
        if (ls[l].d_norm_weight && !aligned(ls[l].d_norm_weight, 16)) return MOE_ERR_ALIGNMENT;
        if ((ff & MOE_F_FORCE_PREFILL) && !A->tc_ok) return MOE_ERR_UNSUPPORTED;
        C.fwd = std::max(C.fwd, ws_layout(A, T, k, ff).total);
        C.Emax = std::max(C.Emax, A->E);
    }
    if ((flags & MOE_F_LOOKAHEAD) && lookahead_smem_bytes(C.Emax) > 200 * 1024)
        return MOE_ERR_UNSUPPORTED;   // the top-k kernel of layers without the decode kernel
    size_t p = align256(C.fwd);
    auto take = [&](size_t bytes) {
        const size_t o = p;
        p = align256(p + bytes);
        return o;
    };
    const size_t xb = (size_t)T * C.H * 4;
    C.xa = take(xb);
    C.xb = take(xb);
    C.xn = take(xb);
    C.out = take(xb);
    C.logits = take((size_t)T * C.Emax * 4);
    C.next = take((size_t)T * C.Emax * 4);
    C.gate = take((size_t)T * 4);
    C.pred = take((size_t)T * k * 4);
    C.total = p;
    return MOE_OK;
}

}  // namespace moe

extern "C" {

moe_status moe_forward_routed(const moe_arena *arena, const float *d_x, int T, int k,
                              const float *d_router, const float *d_gate_row, float *d_logits,
                              float *d_gate, float *d_out, void *d_ws, size_t ws_bytes,
                              uint32_t flags, void *stream) {
    flags &= ~MOE_F_LOOKAHEAD;
    moe_status r = forward_checks(arena, d_x, d_logits, T, k, d_out, d_ws, ws_bytes, flags);
    if (r != MOE_OK) return r;
    if ((r = check_router_rows(arena, d_router, d_gate_row)) != MOE_OK) return r;
    if (d_gate_row && !d_gate) return MOE_ERR_INVALID_ARG;
    if (d_gate && !aligned(d_gate, 4)) return MOE_ERR_ALIGNMENT;
    if ((T + 15) / 16 > 65535) return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    RouterRowsArgs a{};
    a.x = d_x;
    a.Wr = d_router;
    a.E = arena->E;
    a.logits = d_logits;
    a.wg = d_gate_row;
    a.gate = d_gate_row ? d_gate : nullptr;
    a.T = T;
    a.H = arena->H;
    if (launch_router_rows(a, st, false) != cudaSuccess) return MOE_ERR_CUDA;
    return forward_impl(arena, d_x, d_logits, a.gate, T, k, d_out, d_ws, ws_bytes, flags, stream);
}

moe_status moe_chain_workspace_size(const moe_chain_layer *host_layers, int n_layers,
                                    int max_tokens, int k, uint32_t flags, size_t *bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    ChainLayout C;
    const moe_status r = chain_layout(host_layers, n_layers, max_tokens, k, flags, C);
    if (r != MOE_OK) return r;
    *bytes = C.total;
    return MOE_OK;
}

moe_status moe_chain_status(const moe_chain_layer *host_layers, int n_layers, void *d_ws, int T,
                            int k, uint32_t flags, uint32_t **d_status_word) {
    if (!d_ws || !d_status_word) return MOE_ERR_INVALID_ARG;
    ChainLayout C;
    const moe_status r = chain_layout(host_layers, n_layers, T, k, flags, C);
    if (r != MOE_OK) return r;
    // every layer's workspace layout starts with the status word
    *d_status_word = reinterpret_cast<uint32_t *>(
        static_cast<uint8_t *>(d_ws) + ws_layout(host_layers[0].arena, T, k, flags).status);
    return MOE_OK;
}

moe_status moe_chain_forward(const moe_chain_layer *host_layers, int n_layers, const float *d_x,
                             int T, int k, float *d_x_out, void *d_ws, size_t ws_bytes,
                             uint32_t flags, const moe_chain_trace *host_trace, void *stream) {
    ChainLayout C;
    moe_status r = chain_layout(host_layers, n_layers, T, k, flags, C);
    if (r != MOE_OK) return r;
    if (!d_x || !d_x_out || !d_ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(d_x, 16) || !aligned(d_x_out, 16) || !aligned(d_ws, 256)) return MOE_ERR_ALIGNMENT;
    if (ws_bytes < C.total) return MOE_ERR_WORKSPACE;
    const moe_chain_trace tr = host_trace ? *host_trace : moe_chain_trace{};
    const bool look = (flags & MOE_F_LOOKAHEAD) != 0;
    const uint32_t ff = flags & ~MOE_F_LOOKAHEAD;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *ws = static_cast<uint8_t *>(d_ws);
    float *xbuf[2] = {reinterpret_cast<float *>(ws + C.xa), reinterpret_cast<float *>(ws + C.xb)};
    float *xn = reinterpret_cast<float *>(ws + C.xn);
    float *out = reinterpret_cast<float *>(ws + C.out);
    float *logits = reinterpret_cast<float *>(ws + C.logits);
    float *next = reinterpret_cast<float *>(ws + C.next);
    float *gate = reinterpret_cast<float *>(ws + C.gate);
    int32_t *pred = reinterpret_cast<int32_t *>(ws + C.pred);   // ids predicted for layer l+1
    const int H = C.H;
    const size_t xbytes = (size_t)T * H * 4;
    auto copy = [&](void *dst, const void *src, size_t bytes) {
        return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st) == cudaSuccess;
    };
    const float *x = d_x;   // x_l
    for (int l = 0; l < n_layers; l++) {
        const moe_chain_layer &Ly = host_layers[l];
        const moe_arena *A = Ly.arena;
        const bool ahead = look && l + 1 < n_layers;
        RouterRowsArgs a{};
        if (l == 0) {
            a.x = d_x;
        } else {   // x_l = x_{l-1} + out_{l-1}, formed and written by the router pass
            a.x = x;
            a.res = out;
            a.x_out = xbuf[l & 1];
        }
        a.norm = 1;   // the layer reads RMSNorm(x_l), written to xn
        a.eps = MOE_CHAIN_RMS_EPS;
        a.gamma = Ly.d_norm_weight;
        a.xn_out = xn;
        a.Wr = Ly.d_router;
        a.E = A->E;
        a.logits = logits;
        if (ahead) {
            a.Wn = host_layers[l + 1].d_router;
            a.En = host_layers[l + 1].arena->E;
            a.logits_next = next;
        }
        a.wg = Ly.d_gate_row;
        a.gate = Ly.d_gate_row ? gate : nullptr;
        a.T = T;
        a.H = H;
        if (look && l > 0) {   // warm L2 with the experts layer l-1 predicted for this layer
            const size_t mb = std::max((size_t)A->F * A->max_stride01, (size_t)A->H * A->max_stride2);
            a.pf.ids = pred;
            a.pf.n = T * k;
            a.pf.shared = A->shared >= 0 ? 1 : 0;
            a.pf.experts = A->d_experts;
            a.pf.E = A->E;
            a.pf.H = A->H;
            a.pf.F = A->F;
            a.pf.pmax = (int)((mb + kPrefetchPiece - 1) / kPrefetchPiece);
        }
        if (launch_router_rows(a, st, true) != cudaSuccess) return MOE_ERR_CUDA;
        if (l > 0) x = xbuf[l & 1];
        Lookahead look{};
        if (ahead) {   // layer l+1's prediction, from the logits of the pass above
            look.logits = next;
            look.E = host_layers[l + 1].arena->E;
            look.ids_out = pred;
        }
        bool fused = false;
        r = forward_impl(A, xn, logits, a.gate, T, k, out, d_ws, C.fwd, ff, stream,
                         ahead ? &look : nullptr, &fused);
        if (r != MOE_OK) return r;
        if (ahead && !fused &&   // the layer ran without the decode kernel: a kernel of its own
            launch_lookahead(next, T, look.E, k, pred, st) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (ahead && tr.early && !copy(tr.early + (size_t)(l + 1) * T * k, pred, (size_t)T * k * 4))
            return MOE_ERR_CUDA;
        const WsLayout L = ws_layout(A, T, k, ff);
        bool ok = true;
        if (tr.x) ok = ok && copy(tr.x + (size_t)l * T * H, x, xbytes);
        if (tr.xn) ok = ok && copy(tr.xn + (size_t)l * T * H, xn, xbytes);
        if (tr.logits)
            for (int t = 0; t < T && ok; t++)
                ok = copy(tr.logits + ((size_t)l * T + t) * C.Emax, logits + (size_t)t * A->E,
                          (size_t)A->E * 4);
        if (tr.ids) ok = ok && copy(tr.ids + (size_t)l * T * k, ws + L.ids, (size_t)T * k * 4);
        if (tr.w) ok = ok && copy(tr.w + (size_t)l * T * k, ws + L.w, (size_t)T * k * 4);
        if (tr.gate && Ly.d_gate_row) ok = ok && copy(tr.gate + (size_t)l * T, gate, (size_t)T * 4);
        if (tr.out) ok = ok && copy(tr.out + (size_t)l * T * H, out, xbytes);
        if (!ok) return MOE_ERR_CUDA;
    }
    if (launch_residual(x, out, d_x_out, T, H, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (tr.x && !copy(tr.x + (size_t)n_layers * T * H, d_x_out, xbytes)) return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // extern "C"
