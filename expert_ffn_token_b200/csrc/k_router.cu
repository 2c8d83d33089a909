// k_router.cu -- the router and the shared-expert gate, from the fp32 hidden state.
//
// The engine keeps the per-token path, the routers among it, on the GPU ("Strata: a 125B MoE at
// 94 tok/s on a 12 GB Card", "Three architecture facts"); its lookahead runs the next layer's
// router early to predict the experts that will be needed ("Strata - the details", expert
// cache).  Here:
//   moe_router_logits  logits[t][e] = sum_h x[t][h] * Wr[e][h]: one warp per (token, expert)
//                      row pair, 16-byte loads of both rows, fp32 sums reduced by shuffles.
//                      The router rows (E x H fp32) are read once per 16 tokens of a CTA.
//   moe_shared_gate    g[t] = 1 / (1 + exp(-sum_h x[t][h] * wg[h])): one warp per token.
// The sums are fp32 in a fixed order, so results repeat bit for bit; against the exact sums
// they carry the usual fp32 summation error.
#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int kRouterWarps = 8;   // experts per CTA (one warp each)
constexpr int kRouterTok = 16;    // tokens per CTA: each router row is read once per 16 tokens

__device__ __forceinline__ float warp_sum32(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// grid (ceil(E / 8), ceil(T / 16)), 256 threads: warp w computes expert e = 8 bx + w for the
// CTA's tokens; every lane keeps 16 token sums and walks the row in float4 steps.
__global__ void __launch_bounds__(kRouterWarps * 32)
    k_router_logits(const float *__restrict__ x, const float *__restrict__ Wr, int T, int H, int E,
                    float *__restrict__ logits) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * kRouterWarps + warp;
    const int t0 = blockIdx.y * kRouterTok;
    if (e >= E) return;
    const int nt = min(kRouterTok, T - t0);
    const float4 *w4 = reinterpret_cast<const float4 *>(Wr + (size_t)e * H);
    float acc[kRouterTok];
#pragma unroll
    for (int t = 0; t < kRouterTok; t++) acc[t] = 0.f;
    for (int i = lane; i < H / 4; i += 32) {
        const float4 w = __ldg(w4 + i);
#pragma unroll
        for (int t = 0; t < kRouterTok; t++) {
            if (t < nt) {
                const float4 v = __ldg(reinterpret_cast<const float4 *>(x + (size_t)(t0 + t) * H) + i);
                acc[t] = fmaf(v.x, w.x, acc[t]);
                acc[t] = fmaf(v.y, w.y, acc[t]);
                acc[t] = fmaf(v.z, w.z, acc[t]);
                acc[t] = fmaf(v.w, w.w, acc[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < kRouterTok; t++) {
        if (t < nt) {
            const float s = warp_sum32(acc[t]);
            if (lane == 0) logits[(size_t)(t0 + t) * E + e] = s;
        }
    }
}

// grid ceil(T / 8), 256 threads: warp w computes the gate of token 8 bx + w.
__global__ void __launch_bounds__(256)
    k_shared_gate(const float *__restrict__ x, const float *__restrict__ wg, int T, int H,
                  float *__restrict__ gate) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    const float4 *x4 = reinterpret_cast<const float4 *>(x + (size_t)t * H);
    const float4 *g4 = reinterpret_cast<const float4 *>(wg);
    float acc = 0.f;
    for (int i = lane; i < H / 4; i += 32) {
        const float4 v = __ldg(x4 + i), w = __ldg(g4 + i);
        acc = fmaf(v.x, w.x, acc);
        acc = fmaf(v.y, w.y, acc);
        acc = fmaf(v.z, w.z, acc);
        acc = fmaf(v.w, w.w, acc);
    }
    const float s = warp_sum32(acc);
    if (lane == 0) gate[t] = 1.0f / (1.0f + expf(-s));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

}  // namespace moe

extern "C" moe_status moe_router_logits(const float *d_x, int T, int H, const float *d_router,
                                        int E, float *d_logits, void *stream) {
    using namespace moe;
    if (!d_x || !d_router || !d_logits || T <= 0 || H <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
    if (H % 4) return MOE_ERR_INVALID_ARG;
    if (!aligned16(d_x) || !aligned16(d_router) || !aligned4(d_logits)) return MOE_ERR_ALIGNMENT;
    const dim3 grid((E + kRouterWarps - 1) / kRouterWarps, (T + kRouterTok - 1) / kRouterTok);
    if (grid.y > 65535u) return MOE_ERR_UNSUPPORTED;
    k_router_logits<<<grid, kRouterWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(
        d_x, d_router, T, H, E, d_logits);
    note_launches(1);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status moe_shared_gate(const float *d_x, int T, int H, const float *d_gate_row,
                                      float *d_gate, void *stream) {
    using namespace moe;
    if (!d_x || !d_gate_row || !d_gate || T <= 0 || H <= 0) return MOE_ERR_INVALID_ARG;
    if (H % 4) return MOE_ERR_INVALID_ARG;
    if (!aligned16(d_x) || !aligned16(d_gate_row) || !aligned4(d_gate)) return MOE_ERR_ALIGNMENT;
    k_shared_gate<<<(T + 7) / 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(d_x, d_gate_row, T,
                                                                              H, d_gate);
    note_launches(1);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
