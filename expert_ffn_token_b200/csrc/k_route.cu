// k_route.cu -- a1 (Q8_1 activation blocks), a2 (router top-k + softmax over the chosen k) and
// a3 (histogram, exclusive scan, stable token-order permutation, per-expert job list).
//
// Q8_1: "q8_1 activations" of the Strata v0.1.39 release notes (fixes, #606), quantized "once
// per token" (Strata-Sage-A1.5-GGUF, round-2 table).  Per 32 values: amax, d = amax/127 (IEEE
// fp32 division), q = round-half-away(x/d) clamped to +-127, stored fp16(d) and
// fp16(d * sum q); a block with a non-finite value is stored as zeros and flagged.
// Routing: the k of E experts with the largest logits (ties to the lower id), weights = softmax
// over those k logits ("only 10 of them" per token: Strata v0.1.31 README, "How does it work?";
// 10 routed of 512: "Strata: a 125B MoE at 94 tok/s on a 12 GB Card", "Three architecture
// facts").
#include "route_dev.cuh"

namespace moe {

// 256 threads = 32 blocks of 32 values per CTA.
__global__ void __launch_bounds__(256) k_quantize(const float *__restrict__ x, int64_t nblocks,
                                                  int8_t *__restrict__ q, uint16_t *d,
                                                  uint16_t *s, float *dsum, uint32_t *status) {
    const int64_t blk = (int64_t)blockIdx.x * 32 + (threadIdx.x >> 3);
    const int sub = threadIdx.x & 7;
    const bool active = blk < nblocks;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (active) v = __ldg(reinterpret_cast<const float4 *>(x + blk * 32) + sub);
    const int64_t b = active ? blk : 0;
    q8_1_block8(v, active, sub, q + b * 32, d + b, s + b, dsum ? dsum + b : nullptr, status);
}

cudaError_t launch_quantize(const float *x, int64_t nblocks, int8_t *q, uint16_t *d, uint16_t *s,
                            float *dsum, uint32_t *status, cudaStream_t st) {
    if (nblocks <= 0) return cudaSuccess;
    const int64_t grid = (nblocks + 31) / 32;
    k_quantize<<<(unsigned)grid, 256, 0, st>>>(x, nblocks, q, d, s, dsum, status);
    note_launches(1);
    return cudaGetLastError();
}

// Warp per token; 4 warps per CTA; each warp stages its row in shared memory.
__global__ void __launch_bounds__(128) k_topk(const float *__restrict__ logits, int T, int E,
                                              int k, int32_t *ids, float *w, uint32_t *status) {
    extern __shared__ float s_rows[];
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 4 + wid;
    if (t >= T) return;
    float *row = s_rows + (size_t)wid * E;
    const float *src = logits + (size_t)t * E;
    for (int e = lane; e < E; e += 32) row[e] = __ldg(src + e);
    __syncwarp();
    warp_topk(row, E, k, ids + (size_t)t * k, w + (size_t)t * k, status, nullptr);
}

cudaError_t launch_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w,
                        uint32_t *status, cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    const size_t smem = (size_t)4 * E * sizeof(float);
    cudaError_t err = ensure_smem(k_topk, smem);
    if (err != cudaSuccess) return err;
    k_topk<<<(T + 3) / 4, 128, smem, st>>>(logits, T, E, k, ids, w, status);
    note_launches(1);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ a3: grouping

// Per chunk of kChunk tokens: how many of its (token, slot) pairs go to each expert.
__global__ void __launch_bounds__(256) k_hist(const int32_t *__restrict__ ids, int T, int k, int E,
                                              int32_t *chunk_counts) {
    extern __shared__ int s_cnt[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kChunk, t1 = min(T, t0 + kChunk);
    for (int a = t0 * k + threadIdx.x; a < t1 * k; a += blockDim.x) atomicAdd(&s_cnt[ids[a]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        chunk_counts[(size_t)blockIdx.x * E + e] = s_cnt[e];
}

// One CTA: per-expert totals, exclusive offsets, per-chunk write cursors, the job list.
__global__ void __launch_bounds__(1024) k_scan(int T, int k, int E, int n_chunks, int shared,
                                               const int32_t *__restrict__ chunk_counts,
                                               int32_t *chunk_base, int32_t *counts,
                                               int32_t *offsets, Job *jobs, int32_t *njobs) {
    __shared__ int s_tot[kMaxE];
    __shared__ int s_flag[kMaxE];
    __shared__ int s_warp[33];
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int c = 0; c < n_chunks; c++) {
            const int v = chunk_counts[(size_t)c * E + e];
            chunk_base[(size_t)c * E + e] = run;
            run += v;
        }
        s_tot[e] = run;
        s_flag[e] = run > 0;
        counts[e] = run;
    }
    __syncthreads();
    const int total = block_exclusive_scan<1024>(s_tot, E, s_warp);
    const int n_used = block_exclusive_scan<1024>(s_flag, E, s_warp);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int off = s_tot[e];
        offsets[e] = off;
        const int cnt = counts[e];
        for (int c = 0; c < n_chunks; c++) chunk_base[(size_t)c * E + e] += off;
        if (cnt > 0) jobs[s_flag[e]] = Job{e, off, cnt, 0};
    }
    if (threadIdx.x == 0) {
        offsets[E] = total;
        if (shared) jobs[n_used] = Job{E, T * k, T, 1};
        *njobs = n_used + (shared ? 1 : 0);
    }
}

// One warp per chunk: stable placement of the chunk's pairs, in ascending (token, slot).
__global__ void __launch_bounds__(32) k_scatter(const int32_t *__restrict__ ids, int T, int k,
                                                int E, int32_t *chunk_base, int32_t *perm,
                                                int32_t *inv_perm) {
    const int lane = threadIdx.x;
    const int t0 = blockIdx.x * kChunk, t1 = min(T, t0 + kChunk);
    int32_t *base = chunk_base + (size_t)blockIdx.x * E;
    for (int a0 = t0 * k; a0 < t1 * k; a0 += 32) {
        const int a = a0 + lane;
        const bool act = a < t1 * k;
        const int e = act ? ids[a] : -1;
        const unsigned peers = __match_any_sync(kFull, e);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        const int leader = __ffs(peers) - 1;
        int pos = 0;
        if (act) {
            pos = base[e] + rank;
            perm[pos] = a;
            if (inv_perm) inv_perm[a] = pos;
        }
        __syncwarp();
        if (act && lane == leader) base[e] += __popc(peers);
        __syncwarp();
    }
}

cudaError_t launch_group(const int32_t *ids, int T, int k, int E, int shared, int32_t *counts,
                         int32_t *offsets, int32_t *perm, int32_t *inv_perm,
                         int32_t *chunk_counts, int32_t *chunk_base, Job *jobs, int32_t *njobs,
                         cudaStream_t st) {
    const int n_chunks = (T + kChunk - 1) / kChunk;
    k_hist<<<n_chunks, 256, (size_t)E * sizeof(int), st>>>(ids, T, k, E, chunk_counts);
    note_launches(1);
    k_scan<<<1, 1024, 0, st>>>(T, k, E, n_chunks, shared, chunk_counts, chunk_base, counts,
                               offsets, jobs, njobs);
    note_launches(1);
    k_scatter<<<n_chunks, 32, 0, st>>>(ids, T, k, E, chunk_base, perm, inv_perm);
    note_launches(1);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ decode: a1-a3 in one CTA

// T <= kDecodeMaxT tokens: one CTA quantizes x, selects every token's experts, builds counts,
// offsets, the permutation and the job list.  Shared memory: T rows of logits, counts.
__global__ void __launch_bounds__(512) k_route_small(const float *__restrict__ x,
                                                     const float *__restrict__ logits, int T,
                                                     int H, int E, int k, int shared,
                                                     WsLayout L, uint8_t *ws) {
    extern __shared__ float s_rows[];                         // [T][E]
    int *s_cnt = reinterpret_cast<int *>(s_rows + (size_t)T * E);   // [E]
    __shared__ int s_ids[kDecodeMaxT * kMaxK];
    __shared__ int s_warp[33];

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

    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // a1: 64 blocks of 32 per pass
    const int64_t nblocks = (int64_t)T * H / 32;
    for (int64_t b0 = 0; b0 < nblocks; b0 += 64) {
        const int64_t blk = b0 + (threadIdx.x >> 3);
        const int sub = threadIdx.x & 7;
        const bool act = blk < nblocks;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (act) v = __ldg(reinterpret_cast<const float4 *>(x + blk * 32) + sub);
        const int64_t b = act ? blk : 0;
        q8_1_block8(v, act, sub, xq + b * 32, xd + b, xs + b, xsum + b, status);
    }
    // a2: warp t selects token t's experts
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
    if (wid < T) {
        float *row = s_rows + (size_t)wid * E;
        const float *src = logits + (size_t)wid * E;
        for (int e = lane; e < E; e += 32) row[e] = __ldg(src + e);
        __syncwarp();
        int my = 0;
        warp_topk(row, E, k, ids + wid * k, w + wid * k, status, &my);
        if (lane < k) s_ids[wid * k + lane] = my;
    }
    __syncthreads();
    // a3
    const int A = T * k;
    for (int a = threadIdx.x; a < A; a += blockDim.x) atomicAdd(&s_cnt[s_ids[a]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = s_cnt[e];
    __syncthreads();
    const int total = block_exclusive_scan<512>(s_cnt, E, s_warp);
    for (int e = threadIdx.x; e < E; e += blockDim.x) offsets[e] = s_cnt[e];
    if (threadIdx.x == 0) offsets[E] = total;
    for (int a = threadIdx.x; a < A; a += blockDim.x) {
        const int e = s_ids[a];
        int rank = 0;
        for (int b = 0; b < a; b++) rank += s_ids[b] == e;
        const int pos = s_cnt[e] + rank;
        perm[pos] = a;
        inv_perm[a] = pos;
    }
    __syncthreads();
    // job list: experts with at least one pair, ascending id (one warp; A <= 512 pairs)
    if (wid == 0) {
        int n_used = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int cnt = e < E ? counts[e] : 0;   // written by this CTA above
            const unsigned used = __ballot_sync(kFull, cnt > 0);
            if (cnt > 0) {
                const int idx = n_used + __popc(used & ((1u << lane) - 1u));
                jobs[idx] = Job{e, s_cnt[e], cnt, 0};
            }
            n_used += __popc(used);
        }
        if (lane == 0) {
            if (shared) jobs[n_used] = Job{E, A, T, 1};
            *njobs = n_used + (shared ? 1 : 0);
        }
    }
}

cudaError_t launch_route_small(const float *x, const float *logits, int T, int H, int E, int k,
                               int shared, const WsLayout &L, uint8_t *ws, cudaStream_t st) {
    const size_t smem = ((size_t)T * E + E) * sizeof(float);
    cudaError_t err = ensure_smem(k_route_small, smem);
    if (err != cudaSuccess) return err;
    k_route_small<<<1, 512, smem, st>>>(x, logits, T, H, E, k, shared, L, ws);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
