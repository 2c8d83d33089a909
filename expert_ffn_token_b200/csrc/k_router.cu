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
//   k_lookahead     the next layer's top-k of the lookahead logits (the same selection as a2),
//                   then an L2 prefetch (cp.async.bulk.prefetch.L2) of every predicted expert's
//                   packed gate, up and down rows, and of the shared expert's.  The weights live
//                   in HBM, so "warming" means pulling them into the 126 MB L2 while the current
//                   layer runs; a wrong guess costs HBM bandwidth the decode layer leaves idle.
//   k_residual      x_L = x_{L-1} + out_{L-1} after the last layer of a chain.
#include <algorithm>

#include "moe_internal.cuh"
#include "ptx.cuh"
#include "route_dev.cuh"

namespace moe {

namespace {

constexpr int kRowWarps = 4;      // rows per CTA (one warp each)
constexpr int kRowTok = 16;       // tokens per CTA: each row is read once per 16 tokens
constexpr int kLookWarps = 8;     // tokens whose top-k one lookahead CTA computes at a time
constexpr uint32_t kPrefetchChunk = 16384;   // bytes per L2 prefetch instruction

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

// grid (ceil(rows / 4), ceil(T / 16)), 128 threads.  Row r of the launch is router row r
// (r < E), lookahead row r - E (r < E + En) or the gate row.  With `res`, warp 0 of the CTAs of
// blockIdx.x == 0 (row 0) also writes x + res to x_out.  With `norm`, every warp first sums the
// squares of its tokens' rows (the same fixed order in every warp, so every warp gets the same
// bits), the rows are multiplied by 1 / sqrt(mean square + eps) (then by gamma, elementwise)
// before the dots, and row 0's warp writes the normalised rows to xn_out.
__global__ void __launch_bounds__(kRowWarps * 32) k_router_rows(const RouterRowsArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * kRowWarps + warp;
    const int t0 = blockIdx.y * kRowTok;
    const int n_rows = a.E + a.En + (a.wg ? 1 : 0);
    if (r >= n_rows) return;
    const int nt = min(kRowTok, a.T - t0);
    const float *row = r < a.E ? a.Wr + (size_t)r * a.H
                       : r < a.E + a.En ? a.Wn + (size_t)(r - a.E) * a.H
                                        : a.wg;
    const bool write_x = a.res && a.x_out && r == 0;
    const bool write_xn = a.norm && a.xn_out && r == 0;
    float scale[kRowTok];
#pragma unroll
    for (int t = 0; t < kRowTok; t++) scale[t] = 1.0f;
    if (a.norm) {
        float ss[kRowTok];
#pragma unroll
        for (int t = 0; t < kRowTok; t++) ss[t] = 0.f;
        for (int i = lane; i < a.H / 4; i += 32) {
#pragma unroll
            for (int t = 0; t < kRowTok; t++) {
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
        for (int t = 0; t < kRowTok; t++) {
            if (t < nt) {
                const float ms = __fdiv_rn(warp_sum32(ss[t]), (float)a.H);
                scale[t] = __frsqrt_rn(__fadd_rn(ms, a.eps));
            }
        }
    }
    const float4 *w4 = reinterpret_cast<const float4 *>(row);
    float acc[kRowTok];
#pragma unroll
    for (int t = 0; t < kRowTok; t++) acc[t] = 0.f;
    for (int i = lane; i < a.H / 4; i += 32) {
        const float4 w = __ldg(w4 + i);
#pragma unroll
        for (int t = 0; t < kRowTok; t++) {
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
#pragma unroll
    for (int t = 0; t < kRowTok; t++) {
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

// One CTA of 8 warps.  Warp w routes tokens w, w + 8, ... with the a2 top-k on a copy of the
// token's logits in shared memory, marks the chosen experts in a bitmap and (ids_out != null)
// stores the ids.  Then every thread prefetches 16 KB pieces of the marked experts' matrices
// (and the shared expert's, index E, when `shared`): gate and up are F rows, down H rows.
// Only the 16-byte-aligned interior of each matrix is prefetched, so no address leaves it.
__global__ void __launch_bounds__(kLookWarps * 32)
    k_lookahead(const float *__restrict__ logits, int T, int E, int k, int shared,
                const ExpertDev *__restrict__ experts, int H, int F, int32_t *ids_out) {
    extern __shared__ __align__(16) uint8_t smem[];
    float *rows = reinterpret_cast<float *>(smem);                           // [8][E]
    uint32_t *mark = reinterpret_cast<uint32_t *>(rows + (size_t)kLookWarps * E);   // [E/32+1]
    __shared__ int32_t s_ids[kLookWarps][kMaxK];
    __shared__ float s_w[kLookWarps][kMaxK];
    __shared__ int s_list[kMaxK * kDecodeMaxT + 1];
    __shared__ int s_n;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int words = (E + 1 + 31) / 32;
    for (int i = threadIdx.x; i < words; i += blockDim.x) mark[i] = 0u;
    __syncthreads();
    float *row = rows + (size_t)warp * E;
    for (int t = warp; t < T; t += kLookWarps) {
        for (int e = lane; e < E; e += 32) row[e] = logits[(size_t)t * E + e];
        __syncwarp();
        warp_topk(row, E, k, s_ids[warp], s_w[warp], nullptr, nullptr);
        __syncwarp();
        if (lane < k) {
            const int id = s_ids[warp][lane];
            atomicOr(&mark[id >> 5], 1u << (id & 31));
            if (ids_out) ids_out[(size_t)t * k + lane] = id;
        }
        __syncwarp();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int n = 0;
        for (int wd = 0; wd < words; wd++) {
            uint32_t m = mark[wd];
            while (m) {
                const int b = __ffs(m) - 1;
                m &= m - 1;
                s_list[n++] = wd * 32 + b;
            }
        }
        if (shared) s_list[n++] = E;
        s_n = n;
    }
    __syncthreads();
    // (expert, matrix, piece) triples, split over the CTA's threads
    const int n = s_n;
    for (int j = 0; j < 3 * n; j++) {
        const ExpertDev &X = experts[s_list[j / 3]];
        const int m = j % 3;
        const size_t bytes = (size_t)(m < 2 ? F : H) * X.stride[m];
        const uintptr_t b0 = (reinterpret_cast<uintptr_t>(X.m[m]) + 15) & ~uintptr_t(15);
        const uintptr_t b1 = (reinterpret_cast<uintptr_t>(X.m[m]) + bytes) & ~uintptr_t(15);
        if (b1 <= b0) continue;
        const size_t len = b1 - b0;
        const size_t pieces = (len + kPrefetchChunk - 1) / kPrefetchChunk;
        for (size_t p = threadIdx.x; p < pieces; p += blockDim.x) {
            const uintptr_t s = b0 + p * kPrefetchChunk;
            const uint32_t sz = (uint32_t)min((size_t)kPrefetchChunk, (size_t)(b1 - s));
            ptx::prefetch_l2(reinterpret_cast<const void *>(s), sz);
        }
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

cudaError_t launch_router_rows(const RouterRowsArgs &a, cudaStream_t st) {
    const int n_rows = a.E + a.En + (a.wg ? 1 : 0);
    const dim3 grid((n_rows + kRowWarps - 1) / kRowWarps, (a.T + kRowTok - 1) / kRowTok);
    if (grid.y > 65535u) return cudaErrorInvalidValue;
    k_router_rows<<<grid, kRowWarps * 32, 0, st>>>(a);
    note_launches(1);
    return cudaGetLastError();
}

size_t lookahead_smem_bytes(int E) {
    return (size_t)kLookWarps * E * sizeof(float) + ((E + 1 + 31) / 32) * sizeof(uint32_t);
}

cudaError_t launch_lookahead(const float *logits, int T, int E, int k, int shared,
                             const ExpertDev *experts, int H, int F, int32_t *ids_out,
                             cudaStream_t st) {
    if (T > kDecodeMaxT) return cudaErrorInvalidValue;
    const size_t smem = lookahead_smem_bytes(E);
    cudaError_t err = ensure_smem(k_lookahead, smem);
    if (err != cudaSuccess) return err;
    k_lookahead<<<1, kLookWarps * 32, smem, st>>>(logits, T, E, k, shared, experts, H, F, ids_out);
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
    return launch_router_rows(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK
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
    return launch_router_rows(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK
                                                                                    : MOE_ERR_CUDA;
}
