// route_dev.cuh -- device helpers of a1-a3 shared by the routing kernels and the fused decode
// kernel: Q8_1 of one 32-value block, warp top-k with renormalised softmax, block scan.
#pragma once

#include <climits>

#include "moe_internal.cuh"

namespace moe {

constexpr unsigned kFull = 0xffffffffu;

// ------------------------------------------------------------------ a1: Q8_1 of one block

// Q8_1 of the 32-value block held by 8 consecutive lanes (4 values each, lane `sub` holds
// values 4*sub..4*sub+3).  Every lane of the warp must call this (shuffles use the full mask).
__device__ __forceinline__ void q8_1_block8(float4 v, bool active, int sub, int8_t *q,
                                            uint16_t *d16, uint16_t *s16, float *dsum,
                                            uint32_t *status) {
    bool fin = isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
    float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
    for (int o = 4; o >= 1; o >>= 1) {
        a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
        fin = __shfl_xor_sync(kFull, (int)fin, o) && fin;
    }
    const float d = __fdiv_rn(a, 127.0f);
    int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
    if (fin && d != 0.0f) {
        q0 = max(-127, min(127, (int)roundf(__fdiv_rn(v.x, d))));
        q1 = max(-127, min(127, (int)roundf(__fdiv_rn(v.y, d))));
        q2 = max(-127, min(127, (int)roundf(__fdiv_rn(v.z, d))));
        q3 = max(-127, min(127, (int)roundf(__fdiv_rn(v.w, d))));
    }
    int sum = q0 + q1 + q2 + q3;
#pragma unroll
    for (int o = 4; o >= 1; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
    if (!active) return;
    const uint32_t packed = (uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8) |
                            ((uint32_t)(q2 & 0xFF) << 16) | ((uint32_t)(q3 & 0xFF) << 24);
    reinterpret_cast<uint32_t *>(q)[sub] = packed;
    if (sub == 0) {
        if (fin) {
            const __half dh = __float2half_rn(d);
            d16[0] = __half_as_ushort(dh);
            s16[0] = __half_as_ushort(__float2half_rn(__fmul_rn(d, (float)sum)));
            // fp16(d) * sum is exact in fp32 (11 x 12 significant bits)
            if (dsum) dsum[0] = __fmul_rn(__half2float(dh), (float)sum);
        } else {
            d16[0] = 0;
            s16[0] = 0;
            if (dsum) dsum[0] = 0.0f;
            set_status(status, MOE_ERR_NONFINITE);
        }
    }
}

// ------------------------------------------------------------------ a2: top-k of one row

// One warp selects the k largest of row[0..E) (shared memory, overwritten) and writes
// ids_out[0..k), w_out[0..k).  Ties go to the lower id; weights are the softmax over the
// chosen k logits.  Returns the chosen (id, logit) of slot `lane` through the pointers.
__device__ __forceinline__ void warp_topk(float *row, int E, int k, int32_t *ids_out, float *w_out,
                          uint32_t *status, int32_t *my_id_out) {
    const int lane = threadIdx.x & 31;
    bool fin = true;
    for (int e = lane; e < E; e += 32) fin = fin && isfinite(row[e]);
    fin = __all_sync(kFull, fin);
    if (!fin) {
        if (lane < k) {
            ids_out[lane] = lane;
            w_out[lane] = __fdiv_rn(1.0f, (float)k);
            if (my_id_out) *my_id_out = lane;
        }
        if (lane == 0) set_status(status, MOE_ERR_NONFINITE);
        return;
    }
    float my_l = 0.0f;
    int my_id = 0;
    for (int j = 0; j < k; j++) {
        float bv = -INFINITY;
        int bi = INT_MAX;
        for (int e = lane; e < E; e += 32) {     // ascending e: '>' keeps the lower id
            const float v = row[e];
            if (v > bv) {
                bv = v;
                bi = e;
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, o);
            const int oi = __shfl_xor_sync(kFull, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if (lane == j) {
            my_l = bv;
            my_id = bi;
        }
        if (lane == (bi & 31)) row[bi] = -INFINITY;   // taken (every finite logit is larger)
        __syncwarp();
    }
    const float l0 = __shfl_sync(kFull, my_l, 0);
    const float ex = lane < k ? expf(my_l - l0) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
    if (lane < k) {
        ids_out[lane] = my_id;
        w_out[lane] = __fdiv_rn(ex, sum);
        if (my_id_out) *my_id_out = my_id;
    }
}

// Block-wide exclusive scan of s[0..n) in shared memory (NT threads); returns the total.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int *s, int n, int *s_warp) {
    const int per = (n + NT - 1) / NT;
    const int start = min(n, (int)threadIdx.x * per), end = min(n, start + per);
    int local = 0;
    for (int i = start; i < end; i++) local += s[i];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int inc = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc += v;
    }
    if (lane == 31) s_warp[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        const int v = lane < NT / 32 ? s_warp[lane] : 0;
        int inc2 = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(kFull, inc2, o);
            if (lane >= o) inc2 += u;
        }
        if (lane < NT / 32) s_warp[lane] = inc2 - v;
        if (lane == 31) s_warp[32] = inc2;
    }
    __syncthreads();
    int run = s_warp[wid] + inc - local;
    for (int i = start; i < end; i++) {
        const int v = s[i];
        s[i] = run;
        run += v;
    }
    const int total = s_warp[32];
    __syncthreads();
    return total;
}

}  // namespace moe
