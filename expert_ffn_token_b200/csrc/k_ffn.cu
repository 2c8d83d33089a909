// k_ffn.cu -- a4-a7 on CUDA cores: grouped dequant-GEMV over packed Q4_K / Q5_K / Q8_0 / Q5_1
// rows.
//
// Decode on the pages streams each selected expert's rows once with register reductions
// ("decode chain: register reductions, a side stream for the gate projections",
// Strata-Sage-A1.5-GGUF, round-2 table) and packs several tokens that share an expert into one
// pass ("sub-warp expert packing", Strata v0.1.39 release notes, Decode #646).  Here:
//   gate/up  one CTA per (expert job, 32-row tile): every row is read once per job with 128-bit
//            non-allocating loads, dotted (dp4a) with the Q8_1 activations of all the job's
//            tokens, reduced with warp shuffles; h = silu(g) * u is re-quantized to Q8_1 per
//            32-row block in the same CTA.
//   down     decode: one warp per output row runs over every job (expert) of the batch, weights
//            each product by the routing weight and writes out[t][i] once -- deterministic, no
//            atomics.  Large batches: one CTA per (job, 32-row tile) with a weighted
//            scatter-add (or per-slot y plus a gather combine).
// The dequantized weight is d*sc*q - dmin*m (Q4_K/Q5_K), d*q (Q8_0) or d*q + m (Q5_1): for a
// sub-block of 32
// the dot with Q8_1 values xd*qx is  d*sc*xd*sum(q*qx) - dmin*m*(xd*sum qx), where the second
// factor xd*sum(qx) is kept exactly in fp32 per activation block (xsum).
#include "dot.cuh"

namespace moe {

// ------------------------------------------------------------------ a4 + a5: gate/up

// grid (F/32, max_jobs), 256 threads: warp w owns rows r0 + 4w .. r0 + 4w + 3 of the tile.
// Dynamic smem: NT rows of activations (q [H], d [H/32], s [H/32]) + h tile [32][NT].
template <int NT>
__global__ void __launch_bounds__(256) k_gateup(FfnArgs a) {
    const int job_i = blockIdx.y;
    if (job_i >= *a.njobs) return;
    const Job job = a.jobs[job_i];
    const ExpertDev ex = a.experts[job.expert];
    const int H = a.H, nb = H / 32;
    const int r0 = blockIdx.x * 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    extern __shared__ __align__(16) uint8_t smem[];
    int8_t *s_q = reinterpret_cast<int8_t *>(smem);
    float *s_d = reinterpret_cast<float *>(smem + (size_t)NT * H);
    float *s_s = s_d + NT * nb;
    float *s_h = s_s + NT * nb;                      // [32][NT]
    __shared__ int s_tok[NT];

    for (int c0 = 0; c0 < job.n; c0 += NT) {
        const int nt = min(NT, job.n - c0);
        if (threadIdx.x < NT) {
            const int i = c0 + threadIdx.x;
            int t = 0;
            if ((int)threadIdx.x < nt) t = job.shared ? i : a.perm[job.slot0 + i] / a.k;
            s_tok[threadIdx.x] = t;
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < NT * (H / 16); idx += blockDim.x) {
            const int tt = idx / (H / 16), ci = idx % (H / 16);
            int4 v = make_int4(0, 0, 0, 0);
            if (tt < nt) v = __ldg(reinterpret_cast<const int4 *>(a.xq + (size_t)s_tok[tt] * H) + ci);
            reinterpret_cast<int4 *>(s_q + (size_t)tt * H)[ci] = v;
        }
        for (int idx = threadIdx.x; idx < NT * nb; idx += blockDim.x) {
            const int tt = idx / nb, b = idx % nb;
            float dv = 0.f, sv = 0.f;
            if (tt < nt) {
                dv = half_bits_to_float(a.xd[(size_t)s_tok[tt] * nb + b]);
                sv = a.xsum[(size_t)s_tok[tt] * nb + b];
            }
            s_d[idx] = dv;
            s_s[idx] = sv;
        }
        __syncthreads();
        ActRow xr[NT];
#pragma unroll
        for (int t = 0; t < NT; t++) xr[t] = ActRow{s_q + (size_t)t * H, s_d + t * nb, s_s + t * nb};
        for (int rr = 0; rr < 4; rr++) {
            const int rl = warp * 4 + rr;
            const int r = r0 + rl;
            float g[NT], u[NT];
#pragma unroll
            for (int t = 0; t < NT; t++) g[t] = u[t] = 0.f;
            row_parts_fmt<NT>(ex.fmt, ex.m[0] + (size_t)r * ex.stride[0], H, xr, nt, g);
            row_parts_fmt<NT>(ex.fmt, ex.m[1] + (size_t)r * ex.stride[1], H, xr, nt, u);
#pragma unroll
            for (int t = 0; t < NT; t++) {
                g[t] = warp_sum(g[t]);
                u[t] = warp_sum(u[t]);
            }
            if (lane == 0) {
#pragma unroll
                for (int t = 0; t < NT; t++) s_h[rl * NT + t] = silu_mul(g[t], u[t]);
            }
        }
        __syncthreads();
        if (warp < nt) {
            const float hv = s_h[lane * NT + warp];
            const int slot = job.slot0 + c0 + warp;
            if (a.h) a.h[(size_t)slot * a.F + r0 + lane] = hv;
            const int hb = a.hpad / 32;
            q8_1_warp32(hv, a.hq + (size_t)slot * a.hpad + r0, a.hd + (size_t)slot * hb + r0 / 32,
                        a.hs + (size_t)slot * hb + r0 / 32, a.hsum + (size_t)slot * hb + r0 / 32,
                        a.status);
        }
        __syncthreads();
    }
}

// Zero Q8_1(h) blocks in the padded tail [F, hpad) of every slot (the down rows' stored width).
__global__ void k_hpad_zero(int8_t *hq, uint16_t *hd, uint16_t *hs, float *hsum, int slots, int F,
                            int hpad) {
    const int nb_tail = (hpad - F) / 32;
    const int hb = hpad / 32;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < slots * nb_tail;
         i += gridDim.x * blockDim.x) {
        const int s = i / nb_tail, b = F / 32 + i % nb_tail;
        reinterpret_cast<int4 *>(hq + (size_t)s * hpad + b * 32)[0] = make_int4(0, 0, 0, 0);
        reinterpret_cast<int4 *>(hq + (size_t)s * hpad + b * 32)[1] = make_int4(0, 0, 0, 0);
        hd[(size_t)s * hb + b] = 0;
        hs[(size_t)s * hb + b] = 0;
        hsum[(size_t)s * hb + b] = 0.f;
    }
}

cudaError_t launch_hpad_zero(const FfnArgs &a, cudaStream_t st) {
    const int slots = a.T * a.k + a.T;   // upper bound, padded tail only
    if (a.hpad > a.F) {
        k_hpad_zero<<<64, 256, 0, st>>>(a.hq, a.hd, a.hs, a.hsum, slots, a.F, a.hpad);
        note_launches(1);
    }
    return cudaGetLastError();
}

cudaError_t launch_gateup_gemv(const FfnArgs &a, cudaStream_t st) {
    cudaError_t err0 = launch_hpad_zero(a, st);
    if (err0 != cudaSuccess) return err0;
    constexpr int NT = 4;
    const size_t smem = (size_t)NT * a.H + 2 * sizeof(float) * NT * (a.H / 32) +
                        sizeof(float) * 32 * NT;
    cudaError_t err = ensure_smem(k_gateup<NT>, smem);
    if (err != cudaSuccess) return err;
    dim3 grid(a.F / 32, a.max_jobs);
    k_gateup<NT><<<grid, 256, smem, st>>>(a);
    note_launches(1);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ a6 + a7, decode

// One warp per output row i: loops over every job (expert), dots row i of its down matrix with
// Q8_1(h) of the job's slots and accumulates w * y into the slot's token; writes out[t][i].
// NT >= T.  Jobs, slot tokens and slot weights are staged in shared memory.
template <int NT>
__global__ void __launch_bounds__(256) k_down_decode(FfnArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    Job *s_jobs = reinterpret_cast<Job *>(smem);
    const int slots = a.T * a.k + a.T;
    int *s_tok = reinterpret_cast<int *>(s_jobs + a.max_jobs);
    float *s_w = reinterpret_cast<float *>(s_tok + slots);
    const int nj = *a.njobs;
    for (int i = threadIdx.x; i < nj; i += blockDim.x) s_jobs[i] = a.jobs[i];
    for (int s = threadIdx.x; s < a.T * a.k; s += blockDim.x) {
        const int p = a.perm[s];
        s_tok[s] = p / a.k;
        s_w[s] = a.w[p];
    }
    for (int t = threadIdx.x; t < a.T; t += blockDim.x) {
        s_tok[a.T * a.k + t] = t;
        s_w[a.T * a.k + t] = a.gate ? a.gate[t] : 1.0f;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * 8 + warp;
    if (i >= a.H) return;
    const int hb = a.hpad / 32;
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; t++) acc[t] = 0.f;
    for (int u = 0; u < nj; u++) {
        const Job job = s_jobs[u];
        const ExpertDev ex = a.experts[job.expert];
        const uint8_t *row = ex.m[2] + (size_t)i * ex.stride[2];
        if (ex.fmt == MOE_FMT_Q8_0) {
            for (int b = lane; b < (a.F + 31) / 32; b += 32) {
                const Q80Block w = q80_load(row, b);
                for (int s = 0; s < job.n; s++) {
                    const int slot = job.slot0 + s;
                    const float v = q80_dot(w, a.hq + (size_t)slot * a.hpad + 32 * b,
                                            half_bits_to_float(a.hd[(size_t)slot * hb + b]));
                    const int t = s_tok[slot];
                    const float wv = s_w[slot] * v;
#pragma unroll
                    for (int tt = 0; tt < NT; tt++)
                        if (tt == t) acc[tt] += wv;
                }
            }
            continue;
        }
        if (ex.fmt == MOE_FMT_Q5_1) {
            for (int b = lane; b < (a.F + 31) / 32; b += 32) {
                const Q51Block w = q51_load(row, b);
                for (int s = 0; s < job.n; s++) {
                    const int slot = job.slot0 + s;
                    const size_t hbase = (size_t)slot * hb + b;
                    const float v = q51_dot(w, a.hq + (size_t)slot * a.hpad + 32 * b,
                                            half_bits_to_float(a.hd[hbase]), a.hsum[hbase]);
                    const int t = s_tok[slot];
                    const float wv = s_w[slot] * v;
#pragma unroll
                    for (int tt = 0; tt < NT; tt++)
                        if (tt == t) acc[tt] += wv;
                }
            }
            continue;
        }
        const int nsb = (a.F + 255) / 256;
        const int j = lane & 7, c = j >> 1, hh = j & 1;
        if (ex.fmt == MOE_FMT_Q6_K) {
            for (int sb = lane >> 3; sb < nsb; sb += 4) {
                const Q6Lane w = q6_unpack(row + (size_t)sb * kQ6KBytes, j);
                const int kl = sb * 256 + c * 64 + hh * 16;
                const int bl = sb * 8 + 2 * c;
                for (int s = 0; s < job.n; s++) {
                    const int slot = job.slot0 + s;
                    const int8_t *hq = a.hq + (size_t)slot * a.hpad;
                    const size_t hbase = (size_t)slot * hb + bl;
                    const float v = q6_dot(w, *reinterpret_cast<const int4 *>(hq + kl),
                                           *reinterpret_cast<const int4 *>(hq + kl + 32),
                                           half_bits_to_float(a.hd[hbase]),
                                           half_bits_to_float(a.hd[hbase + 1]));
                    const int t = s_tok[slot];
                    const float wv = s_w[slot] * v;
#pragma unroll
                    for (int tt = 0; tt < NT; tt++)
                        if (tt == t) acc[tt] += wv;
                }
            }
            continue;
        }
        const bool q5 = ex.fmt == MOE_FMT_Q5_K;
        const int SBB = q5 ? kQ5KBytes : kQ4KBytes;
        for (int sb = lane >> 3; sb < nsb; sb += 4) {
            const uint8_t *p = row + (size_t)sb * SBB;
            const uint4 hdr = ld_stream16(p);
            const uint4 qv = ld_stream16(p + (q5 ? 48 : 16) + 16 * j);
            uint4 qh = make_uint4(0, 0, 0, 0);
            if (q5) qh = ld_stream16(p + 16 + 16 * hh);
            const KqLane w = q5 ? kq_unpack<MOE_FMT_Q5_K>(hdr, qv, qh, j)
                                : kq_unpack<MOE_FMT_Q4_K>(hdr, qv, qh, j);
            const int kl = sb * 256 + c * 64 + hh * 16;
            const int bl = sb * 8 + 2 * c;
            for (int s = 0; s < job.n; s++) {
                const int slot = job.slot0 + s;
                const int8_t *hq = a.hq + (size_t)slot * a.hpad;
                const int4 xa = *reinterpret_cast<const int4 *>(hq + kl);
                const int4 xb = *reinterpret_cast<const int4 *>(hq + kl + 32);
                const size_t hbase = (size_t)slot * hb + bl;
                const float v = kq_dot(w, hh, xa, xb, half_bits_to_float(a.hd[hbase]),
                                       half_bits_to_float(a.hd[hbase + 1]), a.hsum[hbase],
                                       a.hsum[hbase + 1]);
                const int t = s_tok[slot];
                const float wv = s_w[slot] * v;
#pragma unroll
                for (int tt = 0; tt < NT; tt++)
                    if (tt == t) acc[tt] += wv;
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; t++) {
        const float v = warp_sum(acc[t]);
        if (lane == 0 && t < a.T) a.out[(size_t)t * a.H + i] = v;
    }
}

cudaError_t launch_down_decode(const FfnArgs &a, cudaStream_t st) {
    const int slots = a.T * a.k + a.T;
    const size_t smem = sizeof(Job) * a.max_jobs + (sizeof(int) + sizeof(float)) * slots;
    const int grid = (a.H + 7) / 8;
    cudaError_t err;
#define MOE_DOWN_CASE(N)                                                                     \
    err = ensure_smem(k_down_decode<N>, smem);                                                   \
    if (err != cudaSuccess) return err;                                                      \
    k_down_decode<N><<<grid, 256, smem, st>>>(a);
    if (a.T <= 1) { MOE_DOWN_CASE(1) }
    else if (a.T <= 4) { MOE_DOWN_CASE(4) }
    else { MOE_DOWN_CASE(16) }
#undef MOE_DOWN_CASE
    note_launches(1);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ a6 + a7, large batches

// grid (ceil(H/32), max_jobs): CTA = 32 output rows of one job's down matrix, slots in chunks
// of NT staged in shared memory; each y is weighted and added into out (atomic) or stored
// per slot for the deterministic gather combine.
template <int NT>
__global__ void __launch_bounds__(256) k_down_grouped(FfnArgs a, int deterministic) {
    const int job_i = blockIdx.y;
    if (job_i >= *a.njobs) return;
    const Job job = a.jobs[job_i];
    const ExpertDev ex = a.experts[job.expert];
    const int K = a.hpad, nb = K / 32;
    const int i0 = blockIdx.x * 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    extern __shared__ __align__(16) uint8_t smem[];
    int8_t *s_q = reinterpret_cast<int8_t *>(smem);
    float *s_d = reinterpret_cast<float *>(smem + (size_t)NT * K);
    float *s_s = s_d + NT * nb;
    __shared__ int s_tok[NT];
    __shared__ float s_w[NT];
    const int Kfmt = small_block(ex.fmt) ? ((a.F + 31) / 32) * 32 : ((a.F + 255) / 256) * 256;
    for (int c0 = 0; c0 < job.n; c0 += NT) {
        const int nt = min(NT, job.n - c0);
        if (threadIdx.x < NT) {
            const int slot = job.slot0 + c0 + threadIdx.x;
            int t = 0;
            float wv = 0.f;
            if ((int)threadIdx.x < nt) {
                if (job.shared) {
                    t = c0 + threadIdx.x;
                    wv = a.gate ? a.gate[t] : 1.0f;
                } else {
                    const int p = a.perm[slot];
                    t = p / a.k;
                    wv = a.w[p];
                }
            }
            s_tok[threadIdx.x] = t;
            s_w[threadIdx.x] = wv;
        }
        for (int idx = threadIdx.x; idx < NT * (K / 16); idx += blockDim.x) {
            const int tt = idx / (K / 16), ci = idx % (K / 16);
            int4 v = make_int4(0, 0, 0, 0);
            if (tt < nt)
                v = __ldg(reinterpret_cast<const int4 *>(a.hq + (size_t)(job.slot0 + c0 + tt) * K) + ci);
            reinterpret_cast<int4 *>(s_q + (size_t)tt * K)[ci] = v;
        }
        for (int idx = threadIdx.x; idx < NT * nb; idx += blockDim.x) {
            const int tt = idx / nb, b = idx % nb;
            float dv = 0.f, sv = 0.f;
            if (tt < nt) {
                dv = half_bits_to_float(a.hd[(size_t)(job.slot0 + c0 + tt) * nb + b]);
                sv = a.hsum[(size_t)(job.slot0 + c0 + tt) * nb + b];
            }
            s_d[idx] = dv;
            s_s[idx] = sv;
        }
        __syncthreads();
        ActRow xr[NT];
#pragma unroll
        for (int t = 0; t < NT; t++) xr[t] = ActRow{s_q + (size_t)t * K, s_d + t * nb, s_s + t * nb};
        for (int rr = 0; rr < 4; rr++) {
            const int i = i0 + warp * 4 + rr;
            if (i >= a.H) break;
            float y[NT];
#pragma unroll
            for (int t = 0; t < NT; t++) y[t] = 0.f;
            row_parts_fmt<NT>(ex.fmt, ex.m[2] + (size_t)i * ex.stride[2], Kfmt, xr, nt, y);
#pragma unroll
            for (int t = 0; t < NT; t++) y[t] = warp_sum(y[t]);
            if (lane < nt) {
                float v = 0.f;
#pragma unroll
                for (int t = 0; t < NT; t++)
                    if (t == lane) v = y[t];
                if (deterministic)
                    a.y[(size_t)(job.slot0 + c0 + lane) * a.H + i] = v;
                else
                    atomicAdd(a.out + (size_t)s_tok[lane] * a.H + i, s_w[lane] * v);
            }
        }
        __syncthreads();
    }
}

cudaError_t launch_down_grouped(const FfnArgs &a, bool deterministic, cudaStream_t st) {
    constexpr int NT = 8;
    const size_t smem = (size_t)NT * a.hpad + 2 * sizeof(float) * NT * (a.hpad / 32);
    cudaError_t err = ensure_smem(k_down_grouped<NT>, smem);
    if (err != cudaSuccess) return err;
    dim3 grid((a.H + 31) / 32, a.max_jobs);
    k_down_grouped<NT><<<grid, 256, smem, st>>>(a, deterministic ? 1 : 0);
    note_launches(1);
    return cudaGetLastError();
}

// out[t][i] = sum_j w[t][j] * y[slot(t, j)][i] + y[T*k + t][i], summed in j order.
__global__ void k_combine(FfnArgs a, int shared) {
    const int t = blockIdx.y;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < a.H; i += gridDim.x * blockDim.x) {
        float acc = 0.f;
        for (int j = 0; j < a.k; j++) {
            const int p = t * a.k + j;
            acc = fmaf(a.w[p], a.y[(size_t)a.inv_perm[p] * a.H + i], acc);
        }
        if (shared) acc = fmaf(a.gate ? a.gate[t] : 1.0f, a.y[((size_t)a.T * a.k + t) * a.H + i], acc);
        a.out[(size_t)t * a.H + i] = acc;
    }
}

cudaError_t launch_combine(const FfnArgs &a, bool shared, cudaStream_t st) {
    dim3 grid((a.H + 255) / 256, a.T);
    k_combine<<<grid, 256, 0, st>>>(a, shared ? 1 : 0);
    note_launches(1);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ debug dequant export

// One thread per weight: RN32(RN32(d*sc)*q - RN32(dmin*m)) (K-quants), d*q (Q8_0),
// RN32(d*q + m) (Q5_1; d*q is exact in fp32, so the fused multiply-add rounds once),
// RN32(RN32(d*sc)*(q - 32)) (Q6_K; d*sc is exact).
__global__ void k_dequant(const uint8_t *__restrict__ m, int fmt, int rows, int nblocks,
                          int stride, float *out) {
    const int bw = block_weights(fmt), bb = block_bytes(fmt);
    const int64_t per_row = (int64_t)nblocks * bw;
    const int64_t total = per_row * rows;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = idx / per_row;
        const int n_in_row = (int)(idx % per_row);
        const int b = n_in_row / bw, n = n_in_row % bw;
        const uint8_t *p = m + r * stride + (int64_t)b * bb;
        const uint32_t d16 = p[0] | (p[1] << 8);
        float w;
        if (fmt == MOE_FMT_Q6_K) {
            const int h = n / 128, i = n % 128, g = i / 32, l = i % 32;
            const int lo = (p[64 * h + l + 32 * (g & 1)] >> (g < 2 ? 0 : 4)) & 15;
            const int hi = (p[128 + 32 * h + l] >> (2 * g)) & 3;
            const int sc = (int8_t)p[192 + 8 * h + 2 * g + l / 16];
            const float d1 = __fmul_rn(half_bits_to_float(p[208] | (p[209] << 8)), (float)sc);
            w = __fmul_rn(d1, (float)(lo + 16 * hi - 32));
        } else if (fmt == MOE_FMT_Q8_0) {
            w = __fmul_rn(half_bits_to_float(d16), (float)(int8_t)p[2 + n]);
        } else if (fmt == MOE_FMT_Q5_1) {
            const uint32_t m16 = p[2] | (p[3] << 8);
            const uint32_t qh = p[4] | (p[5] << 8) | (p[6] << 16) | ((uint32_t)p[7] << 24);
            int q = n < 16 ? (p[8 + n] & 15) : (p[8 + n - 16] >> 4);
            q |= (int)((qh >> n) & 1u) << 4;
            w = __fmaf_rn(half_bits_to_float(d16), (float)q, half_bits_to_float(m16));
        } else {
            const uint32_t m16 = p[2] | (p[3] << 8);
            const int c = n / 64, rr = n % 64;
            const int j = rr < 32 ? 2 * c : 2 * c + 1;
            const uint8_t *qs = p + (fmt == MOE_FMT_Q5_K ? 48 : 16);
            int q = rr < 32 ? (qs[32 * c + rr] & 15) : (qs[32 * c + rr - 32] >> 4);
            if (fmt == MOE_FMT_Q5_K) {
                const uint8_t *qh = p + 16;
                q += rr < 32 ? 16 * ((qh[rr] >> (2 * c)) & 1) : 16 * ((qh[rr - 32] >> (2 * c + 1)) & 1);
            }
            uint32_t s0 = p[4] | (p[5] << 8) | (p[6] << 16) | ((uint32_t)p[7] << 24);
            uint32_t s1 = p[8] | (p[9] << 8) | (p[10] << 16) | ((uint32_t)p[11] << 24);
            uint32_t s2 = p[12] | (p[13] << 8) | (p[14] << 16) | ((uint32_t)p[15] << 24);
            int sc, mn;
            kq_scale_min(s0, s1, s2, j, sc, mn);
            const float d1 = __fmul_rn(half_bits_to_float(d16), (float)sc);
            const float m1 = __fmul_rn(half_bits_to_float(m16), (float)mn);
            w = __fmaf_rn(d1, (float)q, -m1);
        }
        out[idx] = w;
    }
}

cudaError_t launch_dequant(const uint8_t *m, int fmt, int rows, int nblocks, int stride,
                           float *out, cudaStream_t st) {
    const int64_t total = (int64_t)rows * nblocks * block_weights(fmt);
    const int grid = (int)std::min<int64_t>((total + 255) / 256, 148 * 16);
    k_dequant<<<grid, 256, 0, st>>>(m, fmt, rows, nblocks, stride, out);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
