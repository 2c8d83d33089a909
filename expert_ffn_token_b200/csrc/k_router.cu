// k_router.cu -- the router, the shared-expert gate and the lookahead expert prefetch, from the
// fp32 hidden state.
//
// The engine keeps the per-token path, the routers among it, on the GPU ("Strata: a 125B MoE at
// 94 tok/s on a 12 GB Card", "Three architecture facts"); its lookahead runs the next layer's
// router early to predict the experts that will be needed and warms them before they are asked
// for ("Strata - the details", expert cache and the STRATA_LOOKAHEAD paragraph).  Here:
//   k_router_rows   one pass over x for up to three sets of fp32 rows: the layer's router rows
//                   (logits), the next layer's router rows (lookahead logits) and the shared
//                   gate row (g = 1 / (1 + exp(-x . wg))).  In a chain of layers the residual
//                   add x_l = x_{l-1} + out_{l-1} and the RMS normalisation of the layer's input
//                   are folded into the same pass: the kernel reads both terms, sums them in fp32,
//                   writes x_l and the normalised rows once and dots the normalised rows with
//                   the router and gate rows.  One warp per (row,
//                   16 tokens); every lane keeps 16 token sums and walks the row in float4
//                   steps, then the warp reduces by shuffles.  The order of every sum is fixed,
//                   so results repeat bit for bit, and one row's sums do not depend on which
//                   other rows the launch computes.
//                   Before the rows, the whole grid issues an L2 prefetch
//                   (cp.async.bulk.prefetch.L2) of the experts predicted for this layer one
//                   layer earlier (and of the shared expert): the weights live in HBM, so
//                   "warming" means pulling them into the 126 MB L2 while this pass runs, ahead
//                   of the layer; a wrong guess costs HBM bandwidth the decode layer leaves idle.
//   k_lookahead     the next layer's top-k of the lookahead logits (the same selection as a2),
//                   for layers that did not run the decode kernel, which predicts inside.
//   k_residual      x_L = x_{L-1} + out_{L-1} after the last layer of a chain.
#include <algorithm>

#include "moe_internal.cuh"
#include "ptx.cuh"
#include "route_dev.cuh"

namespace moe {

namespace {

constexpr int kRowWarps = 4;      // rows per CTA (one warp each)
constexpr int kRowTok = 16;       // most tokens per CTA: each row is read once per 16 tokens
constexpr int kRowUnroll = 4;     // row steps (512 bytes each) whose loads are issued together
constexpr int kLookWarps = 8;     // tokens whose top-k one lookahead CTA computes at a time
constexpr uint32_t kPrefetchChunk = kPrefetchPiece;   // bytes per L2 prefetch instruction

__device__ __forceinline__ float warp_sum32(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Element chunk i (float4) of token row o: x, plus res when given.
__device__ __forceinline__ float4 hidden4(const RouterRowsArgs &a, size_t o, int i) {
    float4 v = __ldg(reinterpret_cast<const float4 *>(a.x + o) + i);
    if (a.res) {
        const float4 q = __ldg(reinterpret_cast<const float4 *>(a.res + o) + i);
        v.x = __fadd_rn(v.x, q.x);
        v.y = __fadd_rn(v.y, q.y);
        v.z = __fadd_rn(v.z, q.z);
        v.w = __fadd_rn(v.w, q.w);
    }
    return v;
}

// grid (ceil(rows / 4), ceil(T / NT)), 128 threads; NT tokens per CTA (1, 2, 4, 8 or 16: the
// smallest that covers T, so that a decode step runs a short loop body).  Row r of the launch is router row r
// (r < E), lookahead row r - E (r < E + En) or the gate row.  With `res`, warp 0 of the CTAs of
// blockIdx.x == 0 (row 0) also writes x + res to x_out.  With `norm`, every warp first sums the
// squares of its tokens' rows (the same fixed order in every warp, so every warp gets the same
// bits), the rows are multiplied by 1 / sqrt(mean square + eps) (then by gamma, elementwise)
// before the dots, and row 0's warp writes the normalised rows to xn_out.
// The grid's share of an expert prefetch: units (id i, matrix m, 16 KB piece p) = (3 i + m) *
// pmax + p, unit u to CTA u mod (number of CTAs), so that every SM issues about the same number
// of pieces.  Only the 16-byte-aligned interior of a matrix is prefetched, so no address leaves
// it.
__device__ __forceinline__ void prefetch_experts(const ExpertPrefetch &f) {
    const int n = f.n + (f.shared ? 1 : 0);
    const int units = 3 * n * f.pmax;
    const int nctas = gridDim.x * gridDim.y;
    for (int u = blockIdx.y * gridDim.x + blockIdx.x + nctas * threadIdx.x; u < units;
         u += nctas * blockDim.x) {
        const int im = u / f.pmax, p = u - im * f.pmax;
        const int i = im / 3, m = im - 3 * i;
        const int e = i < f.n ? f.ids[i] : f.E;
        if (e < 0 || e > f.E || (e == f.E && !f.shared)) continue;
        const ExpertDev &X = f.experts[e];
        const size_t bytes = (size_t)(m < 2 ? f.F : f.H) * X.stride[m];
        const uintptr_t b0 = (reinterpret_cast<uintptr_t>(X.m[m]) + 15) & ~uintptr_t(15);
        const uintptr_t b1 = (reinterpret_cast<uintptr_t>(X.m[m]) + bytes) & ~uintptr_t(15);
        const uintptr_t s = b0 + (uintptr_t)p * kPrefetchChunk;
        if (s >= b1) continue;
        ptx::prefetch_l2(reinterpret_cast<const void *>(s),
                         (uint32_t)min((uintptr_t)kPrefetchChunk, b1 - s));
    }
}

template <int NT>
__global__ void __launch_bounds__(kRowWarps * 32) k_router_rows(const RouterRowsArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * kRowWarps + warp;
    const int t0 = blockIdx.y * NT;
    const int n_rows = a.E + a.En + (a.wg ? 1 : 0);
    const float *row = r >= n_rows ? nullptr
                       : r < a.E ? a.Wr + (size_t)r * a.H
                       : r < a.E + a.En ? a.Wn + (size_t)(r - a.E) * a.H
                                        : a.wg;
    // Launched behind the previous layer (programmatic dependent launch), the pass first pulls
    // its own rows into L2 -- they depend on nothing before it -- and only then waits for the
    // previous grid, whose output (x, res, the predicted ids) it reads.  Launched plainly, the
    // wait returns at once.
    if (row && lane == 0 && blockIdx.y == 0) ptx::prefetch_l2(row, (uint32_t)(a.H * 4));
    ptx::grid_dependency_wait();
    ptx::launch_dependents();
    if (a.pf.ids) prefetch_experts(a.pf);
    if (!row) return;
    const int nt = min(NT, a.T - t0);
    const bool write_x = a.res && a.x_out && r == 0;
    const bool write_xn = a.norm && a.xn_out && r == 0;
    float scale[NT];
#pragma unroll
    for (int t = 0; t < NT; t++) scale[t] = 1.0f;
    if (a.norm) {
        float ss[NT];
#pragma unroll
        for (int t = 0; t < NT; t++) ss[t] = 0.f;
#pragma unroll 4
        for (int i = lane; i < a.H / 4; i += 32) {
#pragma unroll
            for (int t = 0; t < NT; t++) {
                if (t < nt) {
                    const float4 v = hidden4(a, (size_t)(t0 + t) * a.H, i);
                    ss[t] = fmaf(v.x, v.x, ss[t]);
                    ss[t] = fmaf(v.y, v.y, ss[t]);
                    ss[t] = fmaf(v.z, v.z, ss[t]);
                    ss[t] = fmaf(v.w, v.w, ss[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < NT; t++) {
            if (t < nt) {
                const float ms = __fdiv_rn(warp_sum32(ss[t]), (float)a.H);
                scale[t] = __frsqrt_rn(__fadd_rn(ms, a.eps));
            }
        }
    }
    const float4 *w4 = reinterpret_cast<const float4 *>(row);
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; t++) acc[t] = 0.f;
    const int H4 = a.H / 4;
    // the row's loads of kRowUnroll steps are issued together (the row comes from HBM; a step at
    // a time would wait out one memory latency per 512 bytes)
    for (int i0 = lane; i0 < H4; i0 += 32 * kRowUnroll) {
        float4 wv[kRowUnroll];
#pragma unroll
        for (int u = 0; u < kRowUnroll; u++)
            wv[u] = i0 + 32 * u < H4 ? __ldg(w4 + i0 + 32 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < kRowUnroll; u++) {
        const int i = i0 + 32 * u;
        if (i >= H4) break;
        const float4 w = wv[u];
#pragma unroll
        for (int t = 0; t < NT; t++) {
            if (t < nt) {
                const size_t o = (size_t)(t0 + t) * a.H;
                float4 v = hidden4(a, o, i);
                if (write_x) reinterpret_cast<float4 *>(a.x_out + o)[i] = v;
                if (a.norm) {
                    v.x = __fmul_rn(v.x, scale[t]);
                    v.y = __fmul_rn(v.y, scale[t]);
                    v.z = __fmul_rn(v.z, scale[t]);
                    v.w = __fmul_rn(v.w, scale[t]);
                    if (a.gamma) {
                        const float4 g = __ldg(reinterpret_cast<const float4 *>(a.gamma) + i);
                        v.x = __fmul_rn(v.x, g.x);
                        v.y = __fmul_rn(v.y, g.y);
                        v.z = __fmul_rn(v.z, g.z);
                        v.w = __fmul_rn(v.w, g.w);
                    }
                    if (write_xn) reinterpret_cast<float4 *>(a.xn_out + o)[i] = v;
                }
                acc[t] = fmaf(v.x, w.x, acc[t]);
                acc[t] = fmaf(v.y, w.y, acc[t]);
                acc[t] = fmaf(v.z, w.z, acc[t]);
                acc[t] = fmaf(v.w, w.w, acc[t]);
            }
        }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; t++) {
        if (t < nt) {
            const float s = warp_sum32(acc[t]);
            if (lane == 0) {
                const int tt = t0 + t;
                if (r < a.E)
                    a.logits[(size_t)tt * a.E + r] = s;
                else if (r < a.E + a.En)
                    a.logits_next[(size_t)tt * a.En + (r - a.E)] = s;
                else
                    a.gate[tt] = 1.0f / (1.0f + expf(-s));
            }
        }
    }
}

// One CTA of 8 warps: warp w routes tokens w, w + 8, ... with the a2 top-k on a copy of the
// token's logits in shared memory and stores the ids (-1 for a row that is not finite).  The
// chain runs it only when the layer did not take the decode kernel, which predicts inside.
__global__ void __launch_bounds__(kLookWarps * 32)
    k_lookahead(const float *__restrict__ logits, int T, int E, int k, int32_t *ids_out) {
    extern __shared__ __align__(16) uint8_t smem[];
    float *rows = reinterpret_cast<float *>(smem);   // [8][E]
    __shared__ int32_t s_ids[kLookWarps][kMaxK];
    __shared__ float s_w[kLookWarps][kMaxK];
    __shared__ uint32_t s_bad[kLookWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *row = rows + (size_t)warp * E;
    for (int t = warp; t < T; t += kLookWarps) {
        for (int e = lane; e < E; e += 32) row[e] = logits[(size_t)t * E + e];
        if (lane == 0) s_bad[warp] = 0u;
        __syncwarp();
        warp_topk(row, E, k, s_ids[warp], s_w[warp], &s_bad[warp], nullptr);
        __syncwarp();
        if (lane < k) ids_out[(size_t)t * k + lane] = s_bad[warp] ? -1 : s_ids[warp][lane];
        __syncwarp();
    }
}

// x_out = x + res, float4 per thread (n4 = T * H / 4).
__global__ void k_residual(const float4 *__restrict__ x, const float4 *__restrict__ res,
                           float4 *__restrict__ x_out, size_t n4) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
         i += (size_t)gridDim.x * blockDim.x) {
        const float4 v = x[i], q = res[i];
        x_out[i] = make_float4(__fadd_rn(v.x, q.x), __fadd_rn(v.y, q.y), __fadd_rn(v.z, q.z),
                               __fadd_rn(v.w, q.w));
    }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

cudaError_t launch_router_rows(const RouterRowsArgs &a, cudaStream_t st, bool pdl) {
    const int n_rows = a.E + a.En + (a.wg ? 1 : 0);
    const int nt = a.T <= 1 ? 1 : a.T <= 2 ? 2 : a.T <= 4 ? 4 : a.T <= 8 ? 8 : kRowTok;
    const dim3 grid((n_rows + kRowWarps - 1) / kRowWarps, (a.T + nt - 1) / nt);
    if (grid.y > 65535u) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kRowWarps * 32);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t err;
    switch (nt) {
        case 1: err = cudaLaunchKernelEx(&cfg, k_router_rows<1>, a); break;
        case 2: err = cudaLaunchKernelEx(&cfg, k_router_rows<2>, a); break;
        case 4: err = cudaLaunchKernelEx(&cfg, k_router_rows<4>, a); break;
        case 8: err = cudaLaunchKernelEx(&cfg, k_router_rows<8>, a); break;
        default: err = cudaLaunchKernelEx(&cfg, k_router_rows<kRowTok>, a); break;
    }
    if (err != cudaSuccess) return err;
    note_launches(1);
    return cudaGetLastError();
}

size_t lookahead_smem_bytes(int E) { return (size_t)kLookWarps * E * sizeof(float); }

cudaError_t launch_lookahead(const float *logits, int T, int E, int k, int32_t *ids_out,
                             cudaStream_t st) {
    if (T > kDecodeMaxT) return cudaErrorInvalidValue;
    const size_t smem = lookahead_smem_bytes(E);
    cudaError_t err = ensure_smem(k_lookahead, smem);
    if (err != cudaSuccess) return err;
    k_lookahead<<<1, kLookWarps * 32, smem, st>>>(logits, T, E, k, ids_out);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_residual(const float *x, const float *res, float *x_out, int T, int H,
                            cudaStream_t st) {
    const size_t n4 = (size_t)T * H / 4;
    const int grid = (int)std::min<size_t>((n4 + 255) / 256, 4096);
    k_residual<<<grid, 256, 0, st>>>(reinterpret_cast<const float4 *>(x),
                                     reinterpret_cast<const float4 *>(res),
                                     reinterpret_cast<float4 *>(x_out), n4);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe

extern "C" moe_status moe_router_logits(const float *d_x, int T, int H, const float *d_router,
                                        int E, float *d_logits, void *stream) {
    using namespace moe;
    if (!d_x || !d_router || !d_logits || T <= 0 || H <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
    if (H % 4) return MOE_ERR_INVALID_ARG;
    if (!aligned16(d_x) || !aligned16(d_router) || !aligned4(d_logits)) return MOE_ERR_ALIGNMENT;
    if ((T + kRowTok - 1) / kRowTok > 65535) return MOE_ERR_UNSUPPORTED;
    RouterRowsArgs a{};
    a.x = d_x;
    a.Wr = d_router;
    a.E = E;
    a.logits = d_logits;
    a.T = T;
    a.H = H;
    return launch_router_rows(a, static_cast<cudaStream_t>(stream), false) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

extern "C" moe_status moe_shared_gate(const float *d_x, int T, int H, const float *d_gate_row,
                                      float *d_gate, void *stream) {
    using namespace moe;
    if (!d_x || !d_gate_row || !d_gate || T <= 0 || H <= 0) return MOE_ERR_INVALID_ARG;
    if (H % 4) return MOE_ERR_INVALID_ARG;
    if (!aligned16(d_x) || !aligned16(d_gate_row) || !aligned4(d_gate)) return MOE_ERR_ALIGNMENT;
    if ((T + kRowTok - 1) / kRowTok > 65535) return MOE_ERR_UNSUPPORTED;
    RouterRowsArgs a{};
    a.x = d_x;
    a.wg = d_gate_row;
    a.gate = d_gate;
    a.T = T;
    a.H = H;
    return launch_router_rows(a, static_cast<cudaStream_t>(stream), false) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}
