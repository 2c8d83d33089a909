// k_decode.cu -- the whole layer (a1-a7) for small batches in ONE persistent kernel.
//
// Decode is bound by streaming the chosen experts' packed bytes once (the pages' decode chain
// streams expert rows with register reductions, Strata-Sage-A1.5-GGUF round-2 table; the verify
// pass packs the tokens that share an expert, Strata v0.1.39 release notes, Decode #646).  On
// B200 that means megabytes in flight from the first microsecond and as few fixed latencies
// as possible:
//
//   prologue (every CTA, identical results; CTA 0 also stores them in the workspace):
//     logits and x are loaded at once; while warps 0..T-1 select each token's experts
//     (logits held in registers, one redux.sync max + min per pick), the other warps quantize
//     x to Q8_1 in shared memory; one warp then builds counts, offsets, slots and the job list
//     from an expert bitmap (popc prefix sums), and the chosen experts' descriptors are cached.
//   partition: the U * F/32 blocks of 32 gate/up rows go round-robin to the CTAs, so every CTA
//     owns whole Q8_1(h) blocks and quantizes them itself; the H down rows (computed after the
//     barrier by everyone) are cut into equal contiguous ranges.
//   pipeline: one producer thread streams the CTA's rows into a ring of shared-memory stages
//     with bulk async copies (TMA engine, mbarrier byte counts, L2 evict-first) as far ahead
//     as the ring allows; 16 consumer warps compute from shared memory.
//   gate/up: a unit is 16 rows of gate and 16 of up; each warp takes 2 rows, each lane a fixed
//     set of 16-byte quant chunks (activations loaded once per chunk, reused over the rows);
//     h = silu(g) * u goes to shared memory and, once the 32-row block is complete, to Q8_1.
//   down: after every CTA has published its blocks (bounded wait on one counter), all Q8_1(h)
//     rows are staged in shared memory; each warp owns one or two output rows of its CTA's
//     range, its lanes split the (expert, chunk) pairs of those rows, weight each slot's
//     product and keep per-token sums, reduced across the lanes once per row --
//     deterministic, each output element written once.
// Every wait is bounded by %globaltimer and reports MOE_ERR_TIMEOUT instead of hanging.  The
// down phase waits on the gate/up work of every CTA: the grid is one CTA per SM (all resident
// together; a programmatically launched successor starts only once every CTA here has
// started).  The last CTA to pass the grid-wide wait resets the counters.
#include "dot.cuh"
#include "ptx.cuh"
#include "route_dev.cuh"

namespace moe {

namespace {

constexpr int kCW = 16;                      // consumer warps
constexpr int kThreads = (kCW + 1) * 32;     // + one producer warp
constexpr int kRG = 2;                       // gate/up rows per warp per unit
constexpr int kUnitPairs = kRG * kCW / 2;    // 16 gate + 16 up rows per unit
constexpr int kDownRowsMax = 2 * kCW;        // down rows per unit: 1 or 2 per warp

enum { ST_END = 0, ST_GU = 1, ST_DOWN = 2 };

struct StageMeta {
    int kind;   // ST_GU: a job, b first row, c rows      ST_DOWN: a i0, b rows, c j0, d j1, e last
    int a, b, c, d, e, f, g;
};

struct JobX {                // a job with its expert's descriptor, cached in shared memory
    const uint8_t *m[3];
    uint32_t stride[3];
    int fmt, expert, slot0, n;
    short shared;
    short by_n;               // the job in position u of the order by token count, descending
};

struct DecParams {
    const ExpertDev *experts;
    const float *x;
    const float *logits;
    float *out;
    const float *gate;     // optional [T]: the shared expert's weight per token (else 1)
    uint8_t *ws;
    WsLayout L;
    int T, H, F, E, k, shared, hpad;
    int stage_bytes, nstages, max_jobs, slots;
    int keep_h;            // also store fp32 h
    uint64_t wait_ns;      // limit of every bounded wait
    Lookahead look;        // the next layer's prediction (look.logits null: none)
    int o_bar, o_meta, o_xq, o_xd, o_xs, o_jobs, o_stok, o_sw, o_hq, o_hd, o_hs, o_gu, o_h,
        o_acc, o_misc;
    int smem_bytes;
};

// The descriptor table is a copy of the arena's own table into this CTA's shared memory: it
// depends on no other CTA, so its wait keeps a long bound whatever the caller's wait limit.
__device__ __forceinline__ uint64_t desc_wait_ns(const DecParams &P) {
    return P.wait_ns > 50000000ull ? P.wait_ns : 50000000ull;
}

// ------------------------------------------------------------------ chunk-level math
//
// A K-quant row is cut into 16-byte quant chunks p = 8*sb + j (sb super-block, j = 0..7,
// c = j/2, hh = j%2): chunk p holds elements 64c+16hh+[0,16) (low nibbles, sub-block 2c) and
// 64c+32+16hh+[0,16) (high nibbles, sub-block 2c+1) of super-block sb.  A Q8_0 or Q5_1 row is
// cut into its 32-weight blocks (chunk p = block p).

struct ActChunk {            // one token's activations matching one chunk
    int4 xa, xb;             // 16 bytes for the low nibbles, 16 for the high (32-weight blocks:
                             // the block's 32 bytes)
    float dl, dh, sl, sh;    // Q8_1 d and exact d*sum(q) of the two 32-blocks (32-weight
                             // blocks: dl, sl)
};

__device__ __forceinline__ ActChunk load_act(const int8_t *q, const float *d, const float *s,
                                             int p, bool small) {
    ActChunk a;
    if (small) {
        a.xa = *reinterpret_cast<const int4 *>(q + 32 * p);
        a.xb = *reinterpret_cast<const int4 *>(q + 32 * p + 16);
        a.dl = d[p];
        a.sl = s[p];
        a.dh = a.sh = 0.f;
    } else {
        const int sb = p >> 3, j = p & 7, c = j >> 1, hh = j & 1;
        const int kl = sb * 256 + c * 64 + hh * 16;
        const int bl = sb * 8 + 2 * c;
        a.xa = *reinterpret_cast<const int4 *>(q + kl);
        a.xb = *reinterpret_cast<const int4 *>(q + kl + 32);
        // bl is even and K-quant rows hold a multiple of 8 blocks: 8-byte aligned pairs
        const float2 dd = *reinterpret_cast<const float2 *>(d + bl);
        const float2 ss = *reinterpret_cast<const float2 *>(s + bl);
        a.dl = dd.x;
        a.dh = dd.y;
        a.sl = ss.x;
        a.sh = ss.y;
    }
    return a;
}

// Weights of one chunk: unpacked quants and the scales of its two sub-blocks.  The 6-bit
// scale/min pairs are extracted without branches: with c' = c & 1 the needed bytes sit at
// positions 2c', 2c'+1 of the three scale words; c < 2 uses (S[j], S[j+4]) & 63, c >= 2 uses
// the nibbles of S[j+4] with the top two bits of S[j-4] / S[j].
struct WChunk {
    uint32_t lo[4], hi[4];
    float dl, dh, ml, mh;
};

template <bool Q5>
__device__ __forceinline__ WChunk kq_chunk(const uint8_t *sbp, int j) {
    const uint4 hdr = *reinterpret_cast<const uint4 *>(sbp);
    const uint4 qv = *reinterpret_cast<const uint4 *>(sbp + (Q5 ? 48 : 16) + 16 * j);
    const int c = j >> 1;
    const int sh = 16 * (c & 1);
    const uint32_t x0 = hdr.y >> sh, x1 = hdr.z >> sh, x2 = hdr.w >> sh;
    uint32_t sc2, m2;
    if (c < 2) {   // lane-constant: the compiler predicates both forms
        sc2 = x0 & 0x3F3Fu;
        m2 = x1 & 0x3F3Fu;
    } else {
        sc2 = (x2 & 0x0F0Fu) | ((x0 >> 2) & 0x3030u);
        m2 = ((x2 >> 4) & 0x0F0Fu) | ((x1 >> 2) & 0x3030u);
    }
    const float d = half_bits_to_float(hdr.x), dmin = half_bits_to_float(hdr.x >> 16);
    WChunk w;
    w.dl = d * (float)(sc2 & 0xFFu);
    w.dh = d * (float)((sc2 >> 8) & 0xFFu);
    w.ml = dmin * (float)(m2 & 0xFFu);
    w.mh = dmin * (float)((m2 >> 8) & 0xFFu);
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
    uint32_t hw[4] = {0u, 0u, 0u, 0u};
    if (Q5) {
        const uint4 qh = *reinterpret_cast<const uint4 *>(sbp + 16 + 16 * (j & 1));
        hw[0] = qh.x;
        hw[1] = qh.y;
        hw[2] = qh.z;
        hw[3] = qh.w;
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
        w.lo[i] = qw[i] & 0x0F0F0F0Fu;
        w.hi[i] = (qw[i] >> 4) & 0x0F0F0F0Fu;
        if (Q5) {
            w.lo[i] |= ((hw[i] >> (2 * c)) & 0x01010101u) << 4;
            w.hi[i] |= ((hw[i] >> (2 * c + 1)) & 0x01010101u) << 4;
        }
    }
    return w;
}

// A Q6_K chunk (super-block at a 2-byte-aligned address in shared memory): the signed bytes
// q - 32 of its two 16-weight pieces and their scales d*sc; no min term (ml = mh = 0), so
// kq_chunk_dot applies unchanged.
__device__ __forceinline__ WChunk q6_chunk(const uint8_t *sbp, int j) {
    const Q6Lane q = q6_unpack(sbp, j);
    WChunk w;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        w.lo[i] = q.lo[i];
        w.hi[i] = q.hi[i];
    }
    w.dl = q.dl;
    w.dh = q.dh;
    w.ml = w.mh = 0.f;
    return w;
}

// Lane share of sum_k w_k * xhat_k over one chunk.  `mf` is 1 on the lane that adds the two
// sub-blocks' min terms (hh == 0) and 0 on its partner.
__device__ __forceinline__ float kq_chunk_dot(const WChunk &w, const ActChunk &a, float mf) {
    int il = __dp4a((int)w.lo[0], a.xa.x, 0);
    il = __dp4a((int)w.lo[1], a.xa.y, il);
    il = __dp4a((int)w.lo[2], a.xa.z, il);
    il = __dp4a((int)w.lo[3], a.xa.w, il);
    int ih = __dp4a((int)w.hi[0], a.xb.x, 0);
    ih = __dp4a((int)w.hi[1], a.xb.y, ih);
    ih = __dp4a((int)w.hi[2], a.xb.z, ih);
    ih = __dp4a((int)w.hi[3], a.xb.w, ih);
    float r = w.dl * (a.dl * (float)il);
    r = fmaf(w.dh, a.dh * (float)ih, r);
    r = fmaf(-mf * w.ml, a.sl, r);
    r = fmaf(-mf * w.mh, a.sh, r);
    return r;
}

__device__ __forceinline__ float q80_chunk_dot(const uint8_t *blk, const ActChunk &a) {
    const float d = half_bits_to_float((uint32_t)blk[0] | ((uint32_t)blk[1] << 8));
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; i++)
        w[i] = (uint32_t)blk[2 + 4 * i] | ((uint32_t)blk[3 + 4 * i] << 8) |
               ((uint32_t)blk[4 + 4 * i] << 16) | ((uint32_t)blk[5 + 4 * i] << 24);
    int acc = __dp4a((int)w[0], a.xa.x, 0);
    acc = __dp4a((int)w[1], a.xa.y, acc);
    acc = __dp4a((int)w[2], a.xa.z, acc);
    acc = __dp4a((int)w[3], a.xa.w, acc);
    acc = __dp4a((int)w[4], a.xb.x, acc);
    acc = __dp4a((int)w[5], a.xb.y, acc);
    acc = __dp4a((int)w[6], a.xb.z, acc);
    acc = __dp4a((int)w[7], a.xb.w, acc);
    return d * (a.dl * (float)acc);
}

// Q5_1 block (24 bytes, 8-byte aligned): d*xd*sum(q*qx) + m*xs.
__device__ __forceinline__ float q51_chunk_dot(const uint8_t *blk, const ActChunk &a) {
    const uint2 *p = reinterpret_cast<const uint2 *>(blk);
    const Q51Block w = q51_unpack(p[0], p[1], p[2]);
    int acc = __dp4a((int)w.w[0], a.xa.x, 0);
    acc = __dp4a((int)w.w[1], a.xa.y, acc);
    acc = __dp4a((int)w.w[2], a.xa.z, acc);
    acc = __dp4a((int)w.w[3], a.xa.w, acc);
    acc = __dp4a((int)w.w[4], a.xb.x, acc);
    acc = __dp4a((int)w.w[5], a.xb.y, acc);
    acc = __dp4a((int)w.w[6], a.xb.z, acc);
    acc = __dp4a((int)w.w[7], a.xb.w, acc);
    return fmaf(w.d * a.dl, (float)acc, w.m * a.sl);
}

// Format classes the kernel is specialised for: every expert Q4_K, every expert Q5_K, or any.
enum { FK_Q4K = 0, FK_Q5K = 1, FK_ANY = 2 };

// R packed rows of K weights (rows[r], nullptr = skip) against n <= NT activation rows (row t
// at q + act[t]*astride).  The lanes of the warp form 32/lpr groups of lpr lanes; the caller
// gives each group its own rows.  A lane takes chunks p = lane%lpr, +lpr, ...; lane-partial
// sums go to acc[R][NT].
template <int NT, int R, int FK>
__device__ __forceinline__ void rows_dot(int fmt_rt, const uint8_t *const (&rows)[R], int K,
                                         const int8_t *q, const float *d, const float *s,
                                         int astride, const int *act, int n, int lpr,
                                         float (&acc)[R][NT]) {
    const int lane = threadIdx.x & 31;
    const int nchunk = K / 32;
    const int fmt = FK == FK_Q4K ? MOE_FMT_Q4_K : FK == FK_Q5K ? MOE_FMT_Q5_K : fmt_rt;
    const bool q80 = fmt == MOE_FMT_Q8_0, q51 = fmt == MOE_FMT_Q5_1, q5 = fmt == MOE_FMT_Q5_K;
    const bool q6 = fmt == MOE_FMT_Q6_K;
    const bool small = q80 || q51;
    const int SBB = q5 ? kQ5KBytes : kQ4KBytes;
#pragma unroll 2
    for (int p = lane % lpr; p < nchunk; p += lpr) {
        const int sb = p >> 3, j = p & 7;
        const float mf = (j & 1) ? 0.f : 1.f;
        // one activation row: keep its chunk in registers across the rows; several: reload
        // each token's chunk per row from shared memory (saves registers, costs a few loads)
        ActChunk a0;
        if (NT == 1) a0 = load_act(q + (size_t)act[0] * astride, d + act[0] * (astride / 32),
                                   s + act[0] * (astride / 32), p, small);
#pragma unroll
        for (int r = 0; r < R; r++) {
            const uint8_t *row = rows[r];
            if (!row) continue;
            if (FK == FK_ANY && small) {
#pragma unroll
                for (int t = 0; t < NT; t++) {
                    if (t < n) {
                        const ActChunk a = NT == 1 ? a0
                            : load_act(q + (size_t)act[t] * astride, d + act[t] * (astride / 32),
                                       s + act[t] * (astride / 32), p, true);
                        acc[r][t] += q80 ? q80_chunk_dot(row + (size_t)p * kQ80Bytes, a)
                                         : q51_chunk_dot(row + (size_t)p * kQ51Bytes, a);
                    }
                }
            } else {
                const WChunk w = (FK == FK_Q5K || (FK == FK_ANY && q5))
                                     ? kq_chunk<true>(row + (size_t)sb * SBB, j)
                                 : (FK == FK_ANY && q6) ? q6_chunk(row + (size_t)sb * kQ6KBytes, j)
                                                        : kq_chunk<false>(row + (size_t)sb * SBB, j);
#pragma unroll
                for (int t = 0; t < NT; t++) {
                    if (t < n) {
                        const ActChunk a = NT == 1 ? a0
                            : load_act(q + (size_t)act[t] * astride, d + act[t] * (astride / 32),
                                       s + act[t] * (astride / 32), p, false);
                        acc[r][t] += kq_chunk_dot(w, a, mf);
                    }
                }
            }
        }
    }
}

// Q8_1 of one block of x held by 8 lanes, into shared memory (and, on CTA 0, the workspace).
__device__ __noinline__ void quant_x_block(float4 v, bool act, int sub, int b, int8_t *s_xq,
                                           float *s_xd, float *s_xs, uint16_t *g_xd,
                                           uint16_t *g_xs, float *g_xsum, uint32_t *status) {
    uint16_t d16 = 0, s16 = 0;
    float dsum = 0.f;
    q8_1_block8(v, act, sub, s_xq + b * 32, &d16, &s16, &dsum, status);
    if (act && sub == 0) {
        s_xd[b] = half_bits_to_float(d16);
        s_xs[b] = dsum;
        if (g_xd) {
            g_xd[b] = d16;
            g_xs[b] = s16;
            g_xsum[b] = dsum;
        }
    }
}

__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// One warp: the k largest of a logit row held in registers (VPL values per lane, value e at
// lane e%32, slot e/32), descending, ties to the lower id.  Lane j < k gets the j-th choice's
// order key and id.  Returns false (nothing chosen) when the row is not all finite.
template <int VPL>
__device__ __forceinline__ bool topk_select(const float *row, int E, int k, uint32_t &my_key,
                                            int &my_id) {
    const int lane = threadIdx.x & 31;
    uint32_t key[VPL];
    bool fin = true;
#pragma unroll
    for (int i = 0; i < VPL; i++) {
        const int e = lane + 32 * i;
        const float v = e < E ? row[e] : 0.f;
        fin = fin && isfinite(v);
        key[i] = e < E ? order_key(v) : 0u;
    }
    my_key = 0;
    my_id = 0;
    if (!__all_sync(kFullMask, fin)) return false;
    for (int j = 0; j < k; j++) {
        uint32_t bk = 0;
        int bi = 0;
#pragma unroll
        for (int i = 0; i < VPL; i++)
            if (key[i] > bk) {   // strict: the lower slot (lower id) wins ties within a lane
                bk = key[i];
                bi = i;
            }
        const uint32_t m = __reduce_max_sync(kFullMask, bk);
        const uint32_t win = __reduce_min_sync(kFullMask, bk == m ? (uint32_t)(lane + 32 * bi)
                                                                   : 0xFFFFFFFFu);
        if (lane == j) {
            my_key = m;
            my_id = (int)win;
        }
        if ((int)(win & 31u) == lane) {
#pragma unroll
            for (int i = 0; i < VPL; i++)
                if (i == (int)(win >> 5)) key[i] = 0u;
        }
    }
    return true;
}

// One warp: top-k of a logit row (as topk_select) and weights = softmax over the chosen k.
template <int VPL>
__device__ __noinline__ void warp_topk_reg(const float *row, int E, int k, int *ids_out,
                                              float *w_out, uint32_t *status) {
    const int lane = threadIdx.x & 31;
    uint32_t my_key;
    int my_id;
    if (!topk_select<VPL>(row, E, k, my_key, my_id)) {
        if (lane < k) {
            ids_out[lane] = lane;
            w_out[lane] = __fdiv_rn(1.0f, (float)k);
        }
        if (lane == 0) set_status(status, MOE_ERR_NONFINITE);
        return;
    }
    const float l0 = key_value(__shfl_sync(kFullMask, my_key, 0));
    const float ex = lane < k ? expf(key_value(my_key) - l0) : 0.f;
    float sum = ex;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(kFullMask, sum, o);
    if (lane < k) {
        ids_out[lane] = my_id;
        w_out[lane] = __fdiv_rn(ex, sum);
    }
}

// Q8_1 of 32 values held one per lane; lane 0 gets d16, s16, dsum.
__device__ __noinline__ int q8_1_lane(float v, bool &fin, uint16_t &d16, uint16_t &s16,
                                      float &dsum) {
    fin = __all_sync(kFullMask, isfinite(v));
    // the largest |v| as the largest bit pattern (non-negative floats order as unsigned
    // integers; a non-finite block is zeroed below whatever this gives)
    const float a = __uint_as_float(__reduce_max_sync(kFullMask, __float_as_uint(fabsf(v))));
    const float d = __fdiv_rn(a, 127.0f);
    int qi = 0;
    if (fin && d != 0.0f) qi = max(-127, min(127, (int)roundf(__fdiv_rn(v, d))));
    const int sum = __reduce_add_sync(kFullMask, qi);
    if (fin) {
        const __half dh = __float2half_rn(d);
        d16 = __half_as_ushort(dh);
        s16 = __half_as_ushort(__float2half_rn(__fmul_rn(d, (float)sum)));
        dsum = __fmul_rn(__half2float(dh), (float)sum);
    } else {
        qi = 0;
        d16 = s16 = 0;
        dsum = 0.f;
    }
    return qi;
}

// What a CTA shares between its phases: shared-memory and workspace views, sizes, its share of
// the work.  Built once by the kernel and passed to the (inlined) phase functions below.
struct Ctx {
    int8_t *s_xq;
    float *s_xd, *s_xs;
    JobX *s_jobs;
    int *s_stok;
    float *s_sw;
    int8_t *s_hq;
    float *s_hd, *s_hs, *s_h;
    int *s_misc;             // [0] jobs [2] timeout
    uint64_t *full, *empty, *desc_bar;
    StageMeta *meta;
    uint8_t *ring;
    uint8_t *ws;
    uint32_t *status, *ctr;  // ctr: [1] blocks published [2] CTAs finished
    int T, H, F, E, k, U, nb32, n_blk, my_blocks, i_lo, i_hi, hb;
    bool cta0;
};

// Where the prologue keeps the expert descriptor table: in the stage ring, after the routing
// scratch (counts, offsets, bitmap, ids, weights), 16-byte aligned.
__device__ __forceinline__ ExpertDev *desc_table(uint8_t *sm, int E, int T, int k) {
    return reinterpret_cast<ExpertDev *>(sm + (((2 * E + 64 + 2 * T * k) * 4 + 15) / 16) * 16);
}

// a1-a3 for the whole batch (every CTA; CTA 0 also stores the intermediates).
template <int VPL, int TT>
__device__ __forceinline__ void prologue(const DecParams &P, Ctx &C, uint8_t *sm) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const WsLayout &L = P.L;
    uint8_t *ws = P.ws;
    const int T = P.T, H = P.H, E = P.E, k = P.k;
    const bool cta0 = C.cta0;
    uint32_t *status = C.status;
    // scratch in the (still unused) stage ring
    int *s_cnt = reinterpret_cast<int *>(sm);                // [E]
    int *s_off = s_cnt + E;                                  // [E]
    uint32_t *s_bits = reinterpret_cast<uint32_t *>(s_off + E);   // [32]
    int *s_wbase = reinterpret_cast<int *>(s_bits + 32);     // [32]
    int *s_ids = s_wbase + 32;                               // [T*k]
    float *s_wt = reinterpret_cast<float *>(s_ids + T * k);  // [T*k]
    const ExpertDev *s_ex = desc_table(sm, E, T, k);   // filled by the entry's bulk copy
#pragma unroll 1
    for (int e = tid; e < E; e += kThreads) s_cnt[e] = 0;
    if (tid < 32) s_bits[tid] = 0;
    // ---- a2 on warps 0..T-1 (T <= 4), a1 on the rest, at the same time
    const int topk_warps = T <= 4 ? T : 0;
    uint16_t *g_xd = cta0 ? reinterpret_cast<uint16_t *>(ws + L.xd) : nullptr;
    uint16_t *g_xs = reinterpret_cast<uint16_t *>(ws + L.xs);
    float *g_xsum = reinterpret_cast<float *>(ws + L.xsum);
    uint32_t *st = cta0 ? status : nullptr;
    if (warp < topk_warps) {
        warp_topk_reg<VPL>(P.logits + (size_t)warp * E, E, k, s_ids + warp * k, s_wt + warp * k, st);
    } else {
        const int nxb = T * (H / 32);
        const int qt = tid - topk_warps * 32, nq = kThreads - topk_warps * 32;
        const int groups = nq / 8, g0 = qt >> 3, sub = qt & 7;
#pragma unroll 1
        for (int b0 = 0; b0 < nxb; b0 += groups * 4) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; u++) {       // four loads in flight per lane
                const int blk = b0 + g0 + u * groups;
                v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (blk < nxb) v[u] = __ldg(reinterpret_cast<const float4 *>(P.x + (size_t)blk * 32) + sub);
            }
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int blk = b0 + g0 + u * groups;
                const bool act = blk < nxb;
                if (!__any_sync(kFullMask, act)) break;   // blocks ascend with u: none left
                quant_x_block(v[u], act, sub, act ? blk : 0, C.s_xq, C.s_xd, C.s_xs, g_xd, g_xs,
                              g_xsum, st);
            }
        }
    }
    if (topk_warps == 0) {       // larger batches: selection after quantization
        __syncthreads();
#pragma unroll 1
        for (int t = warp; t < T; t += kCW + 1)
            warp_topk_reg<VPL>(P.logits + (size_t)t * E, E, k, s_ids + t * k, s_wt + t * k, st);
    }
    if (T == 1 && k <= 32) {
        // One token: its k experts are distinct, so warp 0 (which chose them) builds the job
        // list in registers -- one job per expert in ascending id, one slot each -- while the
        // other warps finish quantizing x.
        if (warp == 0) {
            const bool v = lane < k;
            const int id = v ? s_ids[lane] : 0x7FFFFFFF;
            int rank = 0;
#pragma unroll 1
            for (int i = 0; i < k; i++) rank += __shfl_sync(kFullMask, id, i) < id ? 1 : 0;
            JobX *jobs = C.s_jobs;
            if (v) {
                JobX &J = jobs[rank];
                J.expert = id;
                J.slot0 = rank;
                J.n = 1;
                J.shared = 0;
                C.s_stok[rank] = 0;
                C.s_sw[rank] = s_wt[lane];
                if (cta0) {
                    reinterpret_cast<int32_t *>(ws + L.ids)[lane] = id;
                    reinterpret_cast<float *>(ws + L.w)[lane] = s_wt[lane];
                    reinterpret_cast<int32_t *>(ws + L.perm)[rank] = lane;
                    reinterpret_cast<int32_t *>(ws + L.inv_perm)[lane] = rank;
                }
            }
            const int U = k + (P.shared ? 1 : 0);
            if (lane == 0) {
                if (P.shared) {
                    JobX &J = jobs[k];
                    J.expert = E;
                    J.slot0 = k;
                    J.n = 1;
                    J.shared = 1;
                }
                C.s_stok[k] = 0;
                C.s_sw[k] = P.gate ? P.gate[0] : 1.0f;
                C.s_misc[0] = U;
            }
            __syncwarp();
            if (!ptx::mbar_wait_bounded(C.desc_bar, 0, desc_wait_ns(P))) {
                if (lane == 0) {   // the table is not there: this CTA does no work
                    set_status(status, MOE_ERR_TIMEOUT);
                    C.s_misc[3] = 1;
                }
            } else
#pragma unroll 1
            for (int u = lane; u < U; u += 32) {
                JobX &J = jobs[u];
                const ExpertDev &ex = s_ex[J.expert];
                J.m[0] = ex.m[0];
                J.m[1] = ex.m[1];
                J.m[2] = ex.m[2];
                J.stride[0] = ex.stride[0];
                J.stride[1] = ex.stride[1];
                J.stride[2] = ex.stride[2];
                J.fmt = ex.fmt;
            }
        }
        __syncthreads();
        if (cta0) {   // the intermediates of a1-a3 in the workspace (from outside the stage
                      // ring: this CTA's producer may already be filling it)
            const int U = C.s_misc[0];
#pragma unroll 1
            for (int i = tid; i < H / 16; i += kThreads)
                reinterpret_cast<int4 *>(ws + L.xq)[i] = reinterpret_cast<const int4 *>(C.s_xq)[i];
#pragma unroll 1
            for (int e = tid; e < E; e += kThreads) {
                int c = 0, o = 0;
#pragma unroll 1
                for (int i = 0; i < k; i++) {
                    const int x = C.s_jobs[i].expert;
                    c += x == e ? 1 : 0;
                    o += x < e ? 1 : 0;
                }
                reinterpret_cast<int32_t *>(ws + L.counts)[e] = c;
                reinterpret_cast<int32_t *>(ws + L.offsets)[e] = o;
            }
            if (tid == 0) reinterpret_cast<int32_t *>(ws + L.offsets)[E] = k;
#pragma unroll 1
            for (int u = tid; u < U; u += kThreads) {
                const JobX &J = C.s_jobs[u];
                reinterpret_cast<Job *>(ws + L.jobs)[u] = Job{J.expert, J.slot0, J.n, J.shared};
            }
            if (tid == 0) *reinterpret_cast<int32_t *>(ws + L.njobs) = U;
        }
        return;
    }
    __syncthreads();
    // ---- a3: counts and an expert bitmap, then one warp builds offsets and jobs
    const int A = T * k;
#pragma unroll 1
    for (int a = tid; a < A; a += kThreads) {
        const int e = s_ids[a];
        atomicAdd(&s_cnt[e], 1);
        atomicOr(&s_bits[e >> 5], 1u << (e & 31));
    }
    if (cta0) {
#pragma unroll 1
        for (int i = tid; i < T * H / 16; i += kThreads)
            reinterpret_cast<int4 *>(ws + L.xq)[i] = reinterpret_cast<const int4 *>(C.s_xq)[i];
#pragma unroll 1
        for (int a = tid; a < A; a += kThreads) {
            reinterpret_cast<int32_t *>(ws + L.ids)[a] = s_ids[a];
            reinterpret_cast<float *>(ws + L.w)[a] = s_wt[a];
        }
    }
    __syncthreads();
    JobX *s_jobs = C.s_jobs;
    if (warp == 0) {
        const int nwords = (E + 31) / 32;
        const uint32_t word = lane < nwords ? s_bits[lane] : 0u;
        int csum = 0;
#pragma unroll 1
        for (uint32_t w = word; w; w &= w - 1) csum += s_cnt[lane * 32 + __ffs(w) - 1];
        int jinc = __popc(word), cinc = csum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(kFullMask, jinc, o), b = __shfl_up_sync(kFullMask, cinc, o);
            if (lane >= o) {
                jinc += a;
                cinc += b;
            }
        }
        int jb = jinc - __popc(word), cb = cinc - csum;
        s_wbase[lane] = cb;
#pragma unroll 1
        for (uint32_t w = word; w; w &= w - 1) {
            const int e = lane * 32 + __ffs(w) - 1;
            const int cnt = s_cnt[e];
            JobX &J = s_jobs[jb++];
            J.expert = e;
            J.slot0 = cb;
            J.n = cnt;
            J.shared = 0;
            s_off[e] = cb;
            cb += cnt;
        }
        const int n_routed = __shfl_sync(kFullMask, jinc, 31);
        if (lane == 0) {
            if (P.shared) {
                JobX &J = s_jobs[n_routed];
                J.expert = E;
                J.slot0 = A;
                J.n = T;
                J.shared = 1;
            }
            C.s_misc[0] = n_routed + (P.shared ? 1 : 0);
        }
    }
    __syncthreads();
    const int U = C.s_misc[0];
    // the slot of assignment a: its expert's offset + the number of earlier assignments of the
    // same expert (token-stable).  Up to 32 assignments one warp finds that rank at once (the
    // lanes holding the same expert, below this lane); more take the plain count.
    if (A <= 32) {
        if (warp == 0) {
            const int e = lane < A ? s_ids[lane] : -1 - lane;   // idle lanes match no one
            const unsigned same = __match_any_sync(kFullMask, e);
            if (lane < A) {
                const int slot = s_off[e] + __popc(same & ((1u << lane) - 1u));
                C.s_stok[slot] = lane / k;
                C.s_sw[slot] = s_wt[lane];
                if (cta0) {
                    reinterpret_cast<int32_t *>(ws + L.perm)[slot] = lane;
                    reinterpret_cast<int32_t *>(ws + L.inv_perm)[lane] = slot;
                }
            }
        }
    } else {
#pragma unroll 1
        for (int a = tid; a < A; a += kThreads) {
            const int e = s_ids[a];
            int rank = 0;
#pragma unroll 1
            for (int b = 0; b < a; b++) rank += s_ids[b] == e;
            const int slot = s_off[e] + rank;
            C.s_stok[slot] = a / k;
            C.s_sw[slot] = s_wt[a];
            if (cta0) {
                reinterpret_cast<int32_t *>(ws + L.perm)[slot] = a;
                reinterpret_cast<int32_t *>(ws + L.inv_perm)[a] = slot;
            }
        }
    }
#pragma unroll 1
    for (int t = tid; t < T; t += kThreads) {
        C.s_stok[A + t] = t;
        C.s_sw[A + t] = P.gate ? P.gate[t] : 1.0f;
    }
    // the jobs by token count, descending (stable): the gate/up blocks are dealt to the CTAs in
    // this order, so that the heavy blocks spread over the grid (multi-token kernels)
    if (TT > 1 && U <= 32) {   // one warp: every job's count against all the others at once
        if (warp == 1) {
            const int n = lane < U ? s_jobs[lane].n : -1;
            int pos = 0;
#pragma unroll
            for (int v = 0; v < 32; v++) {
                const int m = __shfl_sync(kFullMask, n, v);
                pos += (v < U && (m > n || (m == n && v < lane))) ? 1 : 0;
            }
            if (lane < U) s_jobs[pos].by_n = (short)lane;
        }
    } else {
#pragma unroll 1
        for (int u = tid; u < U && TT > 1; u += kThreads) {
            const int n = s_jobs[u].n;
            int pos = 0;
#pragma unroll 1
            for (int v = 0; v < U; v++) {
                const int m = s_jobs[v].n;
                pos += (m > n || (m == n && v < u)) ? 1 : 0;
            }
            s_jobs[pos].by_n = (short)u;
        }
    }
    bool desc_ok = true;
    if (tid < U && !ptx::mbar_wait_bounded(C.desc_bar, 0, desc_wait_ns(P))) {
        desc_ok = false;   // the table is not there: this CTA does no work
        set_status(status, MOE_ERR_TIMEOUT);
        C.s_misc[3] = 1;
    }
#pragma unroll 1
    for (int u = tid; u < U && desc_ok; u += kThreads) {
        JobX &J = s_jobs[u];
        const ExpertDev &ex = s_ex[J.expert];
        J.m[0] = ex.m[0];
        J.m[1] = ex.m[1];
        J.m[2] = ex.m[2];
        J.stride[0] = ex.stride[0];
        J.stride[1] = ex.stride[1];
        J.stride[2] = ex.stride[2];
        J.fmt = ex.fmt;
    }
    if (cta0) {
#pragma unroll 1
        for (int e = tid; e < E; e += kThreads) {
            reinterpret_cast<int32_t *>(ws + L.counts)[e] = s_cnt[e];
            const uint32_t below = s_bits[e >> 5] & ((1u << (e & 31)) - 1u);
            int off = s_wbase[e >> 5];
#pragma unroll 1
            for (uint32_t w = below; w; w &= w - 1) off += s_cnt[(e & ~31) + __ffs(w) - 1];
            reinterpret_cast<int32_t *>(ws + L.offsets)[e] = off;
        }
        if (tid == 0) reinterpret_cast<int32_t *>(ws + L.offsets)[E] = A;
    }
    __syncthreads();
    if (cta0) {
#pragma unroll 1
        for (int u = tid; u < U; u += kThreads) {
            const JobX &J = s_jobs[u];
            reinterpret_cast<Job *>(ws + L.jobs)[u] = Job{J.expert, J.slot0, J.n, J.shared};
        }
        if (tid == 0) *reinterpret_cast<int32_t *>(ws + L.njobs) = U;
    }
}

// Stage ring bookkeeping of the producer.
struct Ring {
    int s;
    uint32_t ph;
};

__device__ __forceinline__ bool ring_acquire(const DecParams &P, const Ctx &C, Ring &R, int &st) {
    if (!ptx::mbar_wait_bounded(&C.empty[R.s], R.ph ^ 1u, P.wait_ns)) return false;
    st = R.s;
    if (++R.s == P.nstages) {
        R.s = 0;
        R.ph ^= 1u;
    }
    return true;
}

// One thread: stream this CTA's gate/up blocks, then its down rows, into the ring.
template <int TT>
__device__ __forceinline__ void producer(const DecParams &P, const Ctx &C) {
    const uint64_t pol = ptx::policy_evict_first();
    Ring R{0, 0u};
    bool ok = true;
    const int G = gridDim.x, cta = blockIdx.x;
    const JobX *s_jobs = C.s_jobs;
#pragma unroll 1
    for (int mb = 0; mb < C.my_blocks && ok; mb++) {
        // multi-token kernels: block i of the order by token count goes to CTA i mod G,
        // serpentine (rounds of G blocks alternate direction), so that every CTA gets a mix of
        // heavy and light blocks; single-token jobs all weigh the same: block i to CTA i mod G
        const int blk = TT > 1 ? mb * G + ((mb & 1) ? G - 1 - cta : cta) : cta + mb * G;
        const int ju = TT > 1 ? s_jobs[blk / C.nb32].by_n : blk / C.nb32, b = blk % C.nb32;
        const JobX &J = s_jobs[ju];
#pragma unroll 1
        for (int half = 0; half < 2 && ok; half++) {
            const int r0 = 32 * b + 16 * half;
            const uint32_t b0 = 16u * J.stride[0], b1 = 16u * J.stride[1];
            int st;
            if (!(ok = ring_acquire(P, C, R, st))) break;
            C.meta[st] = StageMeta{ST_GU, ju, r0, 16, 0, 0, 0, 0};
            uint8_t *dst = C.ring + (size_t)st * P.stage_bytes;
            ptx::mbar_arrive_expect_tx(&C.full[st], b0 + b1);
            ptx::bulk_g2s(dst, J.m[0] + (size_t)r0 * J.stride[0], b0, &C.full[st], pol);
            ptx::bulk_g2s(dst + b0, J.m[1] + (size_t)r0 * J.stride[1], b1, &C.full[st], pol);
        }
    }
    const int down_rows = 32;
#pragma unroll 1
    for (int i = C.i_lo; i < C.i_hi && ok;) {
        const int rows = min(down_rows, C.i_hi - i);
        int j = 0;
#pragma unroll 1
        while (j < C.U && ok) {
            const int j0 = j;
            uint32_t bytes = 0;
#pragma unroll 1
            while (j < C.U) {
                const uint32_t b = (uint32_t)rows * s_jobs[j].stride[2];
                if (j > j0 && bytes + b > (uint32_t)P.stage_bytes) break;
                bytes += b;
                j++;
            }
            int st;
            if (!(ok = ring_acquire(P, C, R, st))) break;
            C.meta[st] = StageMeta{ST_DOWN, i, rows, j0, j, j == C.U ? 1 : 0, 0, 0};
            uint8_t *dst = C.ring + (size_t)st * P.stage_bytes;
            ptx::mbar_arrive_expect_tx(&C.full[st], bytes);
            uint32_t off = 0;
#pragma unroll 1
            for (int jj = j0; jj < j; jj++) {
                const JobX &J = s_jobs[jj];
                const uint32_t b = (uint32_t)rows * J.stride[2];
                ptx::bulk_g2s(dst + off, J.m[2] + (size_t)i * J.stride[2], b, &C.full[st], pol);
                off += b;
            }
        }
        i += rows;
    }
    int st;
    if (ok && ring_acquire(P, C, R, st)) {
        C.meta[st] = StageMeta{ST_END, 0, 0, 0, 0, 0, 0, 0};
        ptx::mbar_arrive(&C.full[st]);
    } else {
        set_status(C.status, MOE_ERR_TIMEOUT);
    }
    // After a wait that ran out the consumers may have left without taking every stage.  The
    // bulk copies already issued land before the CTA leaves: wait (bounded) for the stages
    // filled last, one ring's worth (older stages were consumed, so their phases are complete;
    // after a normal run every one of these waits returns at once).
    Ring B = R;
#pragma unroll 1
    for (int q = 0; q < P.nstages; q++) {
        if (--B.s < 0) {
            B.s = P.nstages - 1;
            B.ph ^= 1u;
        }
        ptx::mbar_wait_bounded(&C.full[B.s], B.ph, 20000000ull);
    }
}

// Q8_1 of a completed 32-row block of h (s_h [32][16]) for every slot of job J.
__device__ __forceinline__ void quantize_h_block(const DecParams &P, const Ctx &C, const JobX &J, int b) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const WsLayout &L = P.L;
    int8_t *g_hq = reinterpret_cast<int8_t *>(P.ws + L.hq);
    uint16_t *g_hd = reinterpret_cast<uint16_t *>(P.ws + L.hd);
    uint16_t *g_hs = reinterpret_cast<uint16_t *>(P.ws + L.hs);
    float *g_hsum = reinterpret_cast<float *>(P.ws + L.hsum);
    float *g_h = reinterpret_cast<float *>(P.ws + L.h);
    const int F = C.F, hb = C.hb, nb32 = C.nb32;
#pragma unroll 1
    for (int t = warp; t < J.n; t += kCW) {
        const int slot = J.slot0 + t;
        const float v = C.s_h[lane * 16 + t];
        if (P.keep_h) g_h[(size_t)slot * F + 32 * b + lane] = v;
        bool fin;
        uint16_t d16, s16;
        float dsum;
        const int q = q8_1_lane(v, fin, d16, s16, dsum);
        g_hq[(size_t)slot * P.hpad + 32 * b + lane] = (int8_t)q;
        if (lane == 0) {
            g_hd[(size_t)slot * hb + b] = d16;
            g_hs[(size_t)slot * hb + b] = s16;
            g_hsum[(size_t)slot * hb + b] = dsum;
            if (!fin) set_status(C.status, MOE_ERR_NONFINITE);
        }
        if (b == nb32 - 1) {   // zero the padded tail [F, hpad) of this slot
#pragma unroll 1
            for (int z = F + lane; z < P.hpad; z += 32) g_hq[(size_t)slot * P.hpad + z] = 0;
#pragma unroll 1
            for (int z = nb32 + lane; z < hb; z += 32) {
                g_hd[(size_t)slot * hb + z] = 0;
                g_hs[(size_t)slot * hb + z] = 0;
                g_hsum[(size_t)slot * hb + z] = 0.f;
            }
        }
    }
}

// After this CTA's gate/up work: wait (bounded) until every block of h is published, then stage
// every slot's Q8_1(h) in shared memory.  Returns false on timeout.
__device__ __forceinline__ bool wait_and_stage_h(const DecParams &P, const Ctx &C,
                                                 uint32_t &arrived) {
    const int ctid = threadIdx.x;
    const WsLayout &L = P.L;
    if (ctid == 0) {
        const uint64_t t0 = ptx::globaltimer();
        int to = 0;
#pragma unroll 1
        while (ptx::ld_acquire_u32(&C.ctr[1]) < (uint32_t)C.n_blk) {
            if (ptx::globaltimer() - t0 > P.wait_ns) {
                to = 1;
                break;
            }
            __nanosleep(32);
        }
        C.s_misc[2] = to;
        if (to) set_status(C.status, MOE_ERR_TIMEOUT);
        // this CTA is past the grid-wide wait: count it.  The CTA that counts last resets both
        // counters for the next launch; its result is read only at the end of the consumer, so
        // the atomic's latency hides behind the down pass.
        arrived = atomicAdd(&C.ctr[2], 1u);
        C.s_misc[5] = 1;
    }
    ptx::named_barrier(1, kCW * 32);
    const int8_t *g_hq = reinterpret_cast<const int8_t *>(P.ws + L.hq);
    const uint16_t *g_hd = reinterpret_cast<const uint16_t *>(P.ws + L.hd);
    const float *g_hsum = reinterpret_cast<const float *>(P.ws + L.hsum);
#pragma unroll 1
    for (int i = ctid; i < P.slots * P.hpad / 16; i += kCW * 32)
        reinterpret_cast<int4 *>(C.s_hq)[i] = ptx::ld_cg_v4(g_hq + (size_t)i * 16);
#pragma unroll 1
    for (int i = ctid; i < P.slots * C.hb; i += kCW * 32) {
        C.s_hd[i] = half_bits_to_float(__ldcg(g_hd + i));
        C.s_hs[i] = __ldcg(g_hsum + i);
    }
    ptx::named_barrier(1, kCW * 32);
    return C.s_misc[2] == 0;
}

// One down stage: rows [0, rows) of the unit (warp w owns rows w and w + 16) times the jobs
// [j0, j1) staged here, job after job, each `rows` rows of its down matrix.  The lanes of a warp
// split the (job, chunk) pairs of a row; each pair is dotted with Q8_1(h) of every slot of its
// job and added, weighted, into the lane's per-token sums.  The order of the sums is fixed, so
// the result is deterministic; the lanes are reduced once, at the end of the unit.
// Chunk p of job J in one down row: its dot with Q8_1(h) of every slot of the job, weighted and
// added into acc[token].
template <int TT, int FK>
__device__ __forceinline__ void down_item(const DecParams &P, const Ctx &C, const uint8_t *row,
                                          const JobX &J, int fmt, int p, float (&acc)[TT]) {
    const int hb = C.hb;
    if (FK == FK_ANY && small_block(fmt)) {
        const bool q80 = fmt == MOE_FMT_Q8_0;
#pragma unroll 1
        for (int t = 0; t < J.n; t++) {
            const int slot = J.slot0 + t;
            const ActChunk a = load_act(C.s_hq + (size_t)slot * P.hpad, C.s_hd + slot * hb,
                                        C.s_hs + slot * hb, p, true);
            const float v = q80 ? q80_chunk_dot(row + (size_t)p * kQ80Bytes, a)
                                : q51_chunk_dot(row + (size_t)p * kQ51Bytes, a);
            const int tok = C.s_stok[slot];
            const float wv = C.s_sw[slot] * v;
#pragma unroll
            for (int tt = 0; tt < TT; tt++)
                if (tt == tok) acc[tt] += wv;
        }
    } else {
        const int SBB = fmt == MOE_FMT_Q5_K ? kQ5KBytes : kQ4KBytes;
        const int sb = p >> 3, j = p & 7;
        const WChunk w = fmt == MOE_FMT_Q5_K ? kq_chunk<true>(row + (size_t)sb * SBB, j)
                         : (FK == FK_ANY && fmt == MOE_FMT_Q6_K)
                             ? q6_chunk(row + (size_t)sb * kQ6KBytes, j)
                             : kq_chunk<false>(row + (size_t)sb * SBB, j);
        const float mf = (j & 1) ? 0.f : 1.f;
        if (TT == 1) {   // one token: every job has exactly one slot (straight-line, so that the
                         // caller's unrolled items overlap)
            const int slot = J.slot0;
            const ActChunk a = load_act(C.s_hq + (size_t)slot * P.hpad, C.s_hd + slot * hb,
                                        C.s_hs + slot * hb, p, false);
            acc[0] += C.s_sw[slot] * kq_chunk_dot(w, a, mf);
        } else {
#pragma unroll 1
            for (int t = 0; t < J.n; t++) {
                const int slot = J.slot0 + t;
                const ActChunk a = load_act(C.s_hq + (size_t)slot * P.hpad, C.s_hd + slot * hb,
                                            C.s_hs + slot * hb, p, false);
                const float v = kq_chunk_dot(w, a, mf);
                const int tok = C.s_stok[slot];
                const float wv = C.s_sw[slot] * v;
#pragma unroll
                for (int tt = 0; tt < TT; tt++)
                    if (tt == tok) acc[tt] += wv;
            }
        }
    }
}

// rows <= kCW + 2 (split; multi-token kernels only): warp w computes row w over every item of the
// stage and, when rows > kCW, its 1/kCW share of the items of the one or two rows past kCW
// (their partial sums are added across warps at the end of the unit, in warp order).  Otherwise
// warp w computes rows w and w + kCW over every item.  (The single-token kernel keeps the plain
// form: code it never runs still costs it instruction fetches.)
template <int TT, int FK>
__device__ __forceinline__ void down_stage(const DecParams &P, const Ctx &C, const uint8_t *stage,
                                           int rows, int j0, int j1, float (&dacc)[2][TT]) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool split = TT > 1 && rows <= kCW + 2;
    const int kq_chunks = P.hpad / 32;          // K-quant rows: 16-byte chunks of 32 weights
    const int sm_chunks = (C.F + 31) / 32;      // Q8_0 / Q5_1 rows: one chunk per block
    uint32_t base = 0;                          // offset of job g0 inside the stage
#pragma unroll 1
    for (int g0 = j0; g0 < j1; g0 += 32) {
        const int ng = min(32, j1 - g0);
        // lane l < ng: job g0 + l -- its bytes in the stage and its chunk count, scanned
        uint32_t sz = 0;
        int nch = 0;
        if (lane < ng) {
            const JobX &J = C.s_jobs[g0 + lane];
            sz = (uint32_t)rows * J.stride[2];
            nch = (FK == FK_ANY && small_block(J.fmt)) ? sm_chunks : kq_chunks;
        }
        uint32_t off = sz;
        int cend = nch;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t a = __shfl_up_sync(kFullMask, off, o);
            const int b = __shfl_up_sync(kFullMask, cend, o);
            if (lane >= o) {
                off += a;
                cend += b;
            }
        }
        off = base + off - sz;                   // exclusive: this lane's job offset
        const int total = __shfl_sync(kFullMask, cend, 31);
#pragma unroll 2
        for (int f0 = 0; f0 < total; f0 += 32) {
            const int f = f0 + lane;
            // the pair (jl, p) of item f
            int jl = 0;
            if (FK != FK_ANY) {
                jl = f / kq_chunks;
            } else {
#pragma unroll 1
                for (int l = 0; l < ng - 1; l++)
                    if (f >= __shfl_sync(kFullMask, cend, l)) jl = l + 1;
            }
            const int cbeg = __shfl_sync(kFullMask, cend - nch, jl & 31);
            const uint32_t joff = __shfl_sync(kFullMask, off, jl & 31);
            if (f >= total) continue;
            const int p = f - cbeg;
            const JobX &J = C.s_jobs[g0 + jl];
            const int fmt = FK == FK_Q4K ? MOE_FMT_Q4_K : FK == FK_Q5K ? MOE_FMT_Q5_K : J.fmt;
#pragma unroll
            for (int rr = 0; rr < 2; rr++) {
                const int r = warp + kCW * rr;
                if (r >= rows || (split && rr > 0)) break;
                down_item<TT, FK>(P, C, stage + joff + (size_t)r * J.stride[2], J, fmt, p, dacc[rr]);
            }
        }
        if (split && rows > kCW) {
            // the rows past kCW: lanes 0-15 take row kCW, lanes 16-31 row kCW + 1, and warp w the
            // items [w * per, (w + 1) * per) of the group; partial sums in dacc[1]
            const int e = lane >> 4, li = lane & 15;
            const int per = (total + kCW - 1) / kCW;
#pragma unroll 1
            for (int q0 = 0; q0 < per; q0 += 16) {
                const int f = warp * per + q0 + li;
                const bool act = q0 + li < per && f < total && kCW + e < rows;
                int jl = 0;
                if (FK != FK_ANY) {
                    jl = f / kq_chunks;
                } else {
#pragma unroll 1
                    for (int l = 0; l < ng - 1; l++)
                        if (f >= __shfl_sync(kFullMask, cend, l)) jl = l + 1;
                }
                const int cbeg = __shfl_sync(kFullMask, cend - nch, jl & 31);
                const uint32_t joff = __shfl_sync(kFullMask, off, jl & 31);
                if (!act) continue;
                const JobX &J = C.s_jobs[g0 + jl];
                const int fmt = FK == FK_Q4K ? MOE_FMT_Q4_K : FK == FK_Q5K ? MOE_FMT_Q5_K : J.fmt;
                down_item<TT, FK>(P, C, stage + joff + (size_t)(kCW + e) * J.stride[2], J, fmt,
                                  f - cbeg, dacc[1]);
            }
        }
        base = __shfl_sync(kFullMask, off + sz, ng - 1);
    }
}

// The 16 consumer warps: gate/up units, then down units, from the ring.
template <int NT, int TT, int FK>
__device__ __forceinline__ void consumer(const DecParams &P, const Ctx &C) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = C.H;
    int s = 0;
    uint32_t ph = 0;
    bool have_h = false, skip_down = false;
    uint32_t arrived = 0;
    float dacc[2][TT];   // down sums of this warp's rows (warp, warp + 16) per token
#pragma unroll 1
    while (true) {
        if (!ptx::mbar_wait_bounded(&C.full[s], ph, P.wait_ns)) {
            if (lane == 0) set_status(C.status, MOE_ERR_TIMEOUT);
            break;
        }
        const StageMeta m = C.meta[s];
        if (m.kind == ST_END) break;
        const uint8_t *stage = C.ring + (size_t)s * P.stage_bytes;
        if (m.kind == ST_GU) {
            // the two halves of a 32-row block go to the two groups of 8 warps, so that the
            // second half is computed while the first still is; warp w8 of the group computes
            // gate and up rows w8 and w8 + 8 of its half, for every token of the job
            const int ju = m.a, r0 = m.b;
            const JobX &J = C.s_jobs[ju];
            const int hrow0 = r0 & 31;   // 0 or 16 inside the block
            const int w8 = warp & 7;
            if ((hrow0 >> 4) == (warp >> 3)) {
                const uint32_t s0 = J.stride[0], s1 = J.stride[1];
                const uint8_t *const rp[4] = {stage + (size_t)w8 * s0, stage + 16u * s0 + (size_t)w8 * s1,
                                              stage + (size_t)(w8 + 8) * s0,
                                              stage + 16u * s0 + (size_t)(w8 + 8) * s1};
#pragma unroll 1
                for (int t0 = 0; t0 < J.n; t0 += NT) {
                    const int n = min(NT, J.n - t0);
                    int act[NT];
#pragma unroll
                    for (int t = 0; t < NT; t++) act[t] = t < n ? C.s_stok[J.slot0 + t0 + t] : 0;
                    float acc[4][NT];
#pragma unroll
                    for (int t = 0; t < NT; t++) acc[0][t] = acc[1][t] = acc[2][t] = acc[3][t] = 0.f;
                    rows_dot<NT, 4, FK>(J.fmt, rp, H, C.s_xq, C.s_xd, C.s_xs, H, act, n, 32, acc);
#pragma unroll
                    for (int t = 0; t < NT; t++) {
                        const float g0 = warp_sum(acc[0][t]), u0 = warp_sum(acc[1][t]);
                        const float g1 = warp_sum(acc[2][t]), u1 = warp_sum(acc[3][t]);
                        if (lane == 0 && t < n) {
                            C.s_h[(hrow0 + w8) * 16 + t0 + t] = silu_mul(g0, u0);
                            C.s_h[(hrow0 + w8 + 8) * 16 + t0 + t] = silu_mul(g1, u1);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&C.empty[s]);
            if (hrow0 == 16) {   // the block is complete: Q8_1 of its 32 rows, per slot
                ptx::named_barrier(1, kCW * 32);
                quantize_h_block(P, C, J, r0 / 32);
                // every slot's Q8_1(h) of this block is written (and s_h is free for the next
                // block): publish the block
                ptx::named_barrier(1, kCW * 32);
                if (threadIdx.x == 0) {
                    __threadfence();
                    atomicAdd(&C.ctr[1], 1u);
                }
            }
        } else {   // ST_DOWN
            if (!have_h) {
                skip_down = !wait_and_stage_h(P, C, arrived);
                have_h = true;
            }
            const int i0 = m.a, rows = m.b;
            if (m.c == 0) {   // first stage of a down unit
#pragma unroll
                for (int rr = 0; rr < 2; rr++)
#pragma unroll
                    for (int t = 0; t < TT; t++) dacc[rr][t] = 0.f;
            }
            if (!skip_down) down_stage<TT, FK>(P, C, stage, rows, m.c, m.d, dacc);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&C.empty[s]);
            if (m.e && !skip_down) {   // last stage of the unit: reduce across the lanes, write
                const bool split = TT > 1 && rows <= kCW + 2;
#pragma unroll
                for (int rr = 0; rr < 2; rr++) {
                    const int r = warp + kCW * rr;
                    if (r >= rows || (split && rr > 0)) break;
#pragma unroll
                    for (int t = 0; t < TT; t++) {
                        if (t >= C.T) break;
                        const float v = warp_sum(dacc[rr][t]);
                        if (lane == 0) P.out[(size_t)t * H + i0 + r] = v;
                    }
                }
                if (split && rows > kCW) {
                    // the rows past kCW: each half-warp's partials into s_h ([kCW][2][TT], free
                    // in the down phase); the last warp to arrive adds them in warp order (no
                    // warp waits for another here)
                    float *part = C.s_h;
#pragma unroll
                    for (int t = 0; t < TT; t++) {
                        float v = dacc[1][t];
#pragma unroll
                        for (int o = 8; o >= 1; o >>= 1) v += __shfl_xor_sync(kFullMask, v, o);
                        if ((lane & 15) == 0) part[(warp * 2 + (lane >> 4)) * TT + t] = v;
                    }
                    __threadfence_block();
                    __syncwarp();
                    int last = 0;
                    if (lane == 0) last = atomicAdd(&C.s_misc[8], 1) == kCW - 1;
                    last = __shfl_sync(kFullMask, last, 0);
                    if (last) {
                        __threadfence_block();
                        const int e = lane >> 4, t = lane & 15;
                        if (kCW + e < rows && t < C.T) {
                            float v = 0.f;
#pragma unroll 1
                            for (int w = 0; w < kCW; w++) v += part[(w * 2 + e) * TT + t];
                            P.out[(size_t)t * H + i0 + kCW + e] = v;
                        }
                        if (lane == 0) C.s_misc[8] = 0;
                    }
                }
            }
        }
        if (++s == P.nstages) {
            s = 0;
            ph ^= 1u;
        }
    }
    if (threadIdx.x == 0 && have_h && arrived == gridDim.x - 1) {
        C.ctr[1] = 0;
        C.ctr[2] = 0;
    }
}

// The router lookahead of a chain, inside the layer: on CTA 0, warp (kCW - 1 - t) takes token
// t's top-k of the next layer's logits (the same selection as a2) and stores the predicted ids;
// the next layer's router pass prefetches those experts into L2 before the next layer runs.  A
// row of logits that is not finite predicts id -1 (nothing is prefetched for it; the next layer
// reports the row).
template <int VPL>
__device__ __noinline__ void lookahead(const float *logits, int E, int k, int32_t *ids_out, int t) {
    const int lane = threadIdx.x & 31;
    uint32_t key;
    int id;
    const bool ok = topk_select<VPL>(logits + (size_t)t * E, E, k, key, id);
    if (lane < k) ids_out[t * k + lane] = ok ? id : -1;
}

// NT: activation rows per pass of rows_dot; TT: largest token count the down sums hold;
// FK: format class of the arena; VPL: router logits per lane (E <= 32 * VPL); LOOK: the chain's
// lookahead is compiled in (a separate instantiation: its code alone costs the plain layer half a
// microsecond of register allocation).
template <int NT, int TT, int FK, int VPL, bool LOOK>
__global__ void __launch_bounds__(kThreads, 1) k_decode_fused(const DecParams P) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5;
    Ctx C;
    C.s_xq = reinterpret_cast<int8_t *>(sm + P.o_xq);
    C.s_xd = reinterpret_cast<float *>(sm + P.o_xd);
    C.s_xs = reinterpret_cast<float *>(sm + P.o_xs);
    C.s_jobs = reinterpret_cast<JobX *>(sm + P.o_jobs);
    C.s_stok = reinterpret_cast<int *>(sm + P.o_stok);
    C.s_sw = reinterpret_cast<float *>(sm + P.o_sw);
    C.s_hq = reinterpret_cast<int8_t *>(sm + P.o_hq);
    C.s_hd = reinterpret_cast<float *>(sm + P.o_hd);
    C.s_hs = reinterpret_cast<float *>(sm + P.o_hs);
    C.s_h = reinterpret_cast<float *>(sm + P.o_h);
    C.s_misc = reinterpret_cast<int *>(sm + P.o_misc);
    C.full = reinterpret_cast<uint64_t *>(sm + P.o_bar);
    C.empty = C.full + P.nstages;
    C.desc_bar = C.full + 32;
    C.meta = reinterpret_cast<StageMeta *>(sm + P.o_meta);
    C.ring = sm;
    C.ws = P.ws;
    C.status = reinterpret_cast<uint32_t *>(P.ws + P.L.status);
    C.ctr = reinterpret_cast<uint32_t *>(P.ws + P.L.sync);
    C.T = P.T;
    C.H = P.H;
    C.F = P.F;
    C.E = P.E;
    C.k = P.k;
    C.cta0 = blockIdx.x == 0;
    C.hb = P.hpad / 32;
    C.nb32 = P.F / 32;

    if (tid == 0) {
#pragma unroll 1
        for (int s = 0; s < P.nstages; s++) {
            ptx::mbar_init(&C.full[s], 1);
            ptx::mbar_init(&C.empty[s], kCW);
        }
        ptx::mbar_init(C.desc_bar, 1);
        ptx::fence_barrier_init();
        C.s_misc[2] = 0;
        C.s_misc[3] = 0;
        C.s_misc[5] = 0;
        C.s_misc[8] = 0;
        // the descriptor table is the arena's (not written by the previous kernel): fetch it
        // now, in the background, before waiting for the previous grid
        const uint32_t nb = (uint32_t)((P.E + P.shared) * sizeof(ExpertDev));
        ptx::mbar_arrive_expect_tx(C.desc_bar, nb);
        ptx::bulk_g2s(desc_table(sm, P.E, P.T, P.k), P.experts, nb, C.desc_bar,
                      ptx::policy_evict_last());
    }
    ptx::grid_dependency_wait();
    ptx::launch_dependents();
    prologue<VPL, TT>(P, C, sm);
    // the prologue scratch in the stage ring is dead from here on
    const int G = gridDim.x, cta = blockIdx.x;
    C.U = C.s_misc[0];
    C.n_blk = C.U * C.nb32;
    if (TT > 1) {
        C.my_blocks = 0;
#pragma unroll 1
        for (int r = 0; r * G < C.n_blk; r++)
            C.my_blocks += r * G + ((r & 1) ? G - 1 - cta : cta) < C.n_blk ? 1 : 0;
    } else {
        C.my_blocks = C.n_blk / G + (cta < C.n_blk % G ? 1 : 0);
    }
    // down rows: computed after the barrier by every CTA, so split evenly
    C.i_lo = (int)((long long)P.H * cta / G);
    C.i_hi = (int)((long long)P.H * (cta + 1) / G);

    if (LOOK && P.look.logits && C.cta0 && warp < kCW && warp >= kCW - P.T)
        lookahead<VPL>(P.look.logits, P.look.E, P.k, P.look.ids_out, kCW - 1 - warp);
    if (C.s_misc[3]) {
        // the descriptor table did not arrive in time: no work here (this CTA's blocks are never
        // published, so the grid-wide waits of the others give up too); the copy lands first
        if (tid == 0) ptx::mbar_wait_bounded(C.desc_bar, 0, 50000000ull);
    } else if (warp == kCW) {
        if ((tid & 31) == 0) producer<TT>(P, C);
    } else {
        consumer<NT, TT, FK>(P, C);
    }
    // A CTA that never reached the grid-wide wait (no down rows, or an early timeout) is
    // counted here.  Its blocks were published before: either some other CTA saw all of them
    // at the wait before counting, or this is the last CTA and all the others did.
    if (tid == 0 && C.s_misc[5] == 0) {
        if (atomicAdd(&C.ctr[2], 1u) == gridDim.x - 1) {
            C.ctr[1] = 0;
            C.ctr[2] = 0;
        }
    }
}

template <int NT, int TT, int FK, int VPL, bool LOOK>
cudaError_t launch_one(const cudaLaunchConfig_t &cfg, const DecParams &P) {
    cudaError_t err = ensure_smem(k_decode_fused<NT, TT, FK, VPL, LOOK>, (size_t)P.smem_bytes);
    if (err != cudaSuccess) return err;
    return cudaLaunchKernelEx(&cfg, k_decode_fused<NT, TT, FK, VPL, LOOK>, P);
}

template <int NT, int TT, int FK, bool LOOK = false>
cudaError_t launch_vpl(const cudaLaunchConfig_t &cfg, const DecParams &P, int E) {
    if (E <= 256) return launch_one<NT, TT, FK, 8, LOOK>(cfg, P);
    if (E <= 512) return launch_one<NT, TT, FK, 16, LOOK>(cfg, P);
    return launch_one<NT, TT, FK, 32, LOOK>(cfg, P);
}

template <int NT, int TT, bool LOOK = false>
cudaError_t launch_fk(const cudaLaunchConfig_t &cfg, const DecParams &P, int fk, int E) {
    if (fk == FK_Q4K) return launch_vpl<NT, TT, FK_Q4K, LOOK>(cfg, P, E);
    if (fk == FK_Q5K) return launch_vpl<NT, TT, FK_Q5K, LOOK>(cfg, P, E);
    return launch_vpl<NT, TT, FK_ANY, LOOK>(cfg, P, E);
}

// Instantiations: batch class (1, <= 4, <= 16 tokens) x format class x top-k width, and the
// single-token class again with the chain's lookahead.  The largest batch class exists only for
// the any-format kernel, to bound the code size.
cudaError_t launch_variant(const cudaLaunchConfig_t &cfg, const DecParams &P, int T, int fk, int E) {
    if (T <= 1 && P.look.logits) return launch_fk<1, 1, true>(cfg, P, fk, E);
    if (T <= 1) return launch_fk<1, 1>(cfg, P, fk, E);
    if (T <= 4) return launch_fk<4, 4>(cfg, P, fk, E);
    return launch_vpl<4, 16, FK_ANY>(cfg, P, E);
}

}  // namespace

cudaError_t launch_decode_fused(const FfnArgs &a, int E, int shared, const float *x,
                                const float *logits, uint8_t *ws, const WsLayout &L,
                                size_t sync_off, size_t blkcnt_off, bool pdl, cudaStream_t st,
                                bool *taken, bool *look_fused) {
    (void)sync_off;
    (void)blkcnt_off;
    *taken = false;
    *look_fused = false;
    if (a.T > kDecodeMaxT || E > 1024 || a.T * a.k > kDecodeMaxT * kMaxK || a.F % 32) return cudaSuccess;
    int dev = 0, nsm = 0, cap = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&cap, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
        return err;
    const int max_s01 = a.max_stride01, max_s2 = a.max_stride2;
    if (max_s01 <= 0 || max_s2 <= 0 || 2 * kUnitPairs * max_s01 > 96 * 1024 ||
        kDownRowsMax * max_s2 > 96 * 1024)
        return cudaSuccess;   // rows too wide for the ring: not taken
    DecParams P{};
    P.experts = a.experts;
    P.x = x;
    P.logits = logits;
    P.out = a.out;
    P.gate = a.gate;
    P.ws = ws;
    P.L = L;
    P.T = a.T;
    P.H = a.H;
    P.F = a.F;
    P.E = E;
    P.k = a.k;
    P.shared = shared;
    P.hpad = a.hpad;
    P.max_jobs = a.max_jobs;
    P.slots = a.T * a.k + a.T;
    P.keep_h = a.h != nullptr;
    P.wait_ns = a.wait_ns;
    // the lookahead runs inside (single-token batches) when the next layer's logits fit this
    // kernel's top-k width
    const int top_width = E <= 256 ? 256 : E <= 512 ? 512 : 1024;
    if (a.look.logits && a.look.ids_out && a.look.E <= top_width && a.T <= 1) P.look = a.look;
    auto al = [](int v, int q) { return (v + q - 1) / q * q; };
    const int fk = a.fmt_mask == (1 << MOE_FMT_Q4_K) ? FK_Q4K
                   : a.fmt_mask == (1 << MOE_FMT_Q5_K) ? FK_Q5K : FK_ANY;
    P.stage_bytes = al(std::max(2 * kUnitPairs * max_s01, kDownRowsMax * max_s2), 1024);
    const int slots = P.slots;
    const int sizes[] = {
        2 * 16 * 8 + 16,                             // barriers (<= 16 stages) + descriptors
        16 * (int)sizeof(StageMeta),                 // stage meta
        al(a.T * a.H, 128),                          // xq
        al(a.T * (a.H / 32) * 4, 16),                // xd
        al(a.T * (a.H / 32) * 4, 16),                // xs
        al(a.max_jobs * (int)sizeof(JobX), 16),      // jobs
        al(slots * 4, 16),                           // slot tokens
        al(slots * 4, 16),                           // slot weights
        al(slots * a.hpad, 128),                     // Q8_1(h) q
        al(slots * (a.hpad / 32) * 4, 16),           // Q8_1(h) d
        al(slots * (a.hpad / 32) * 4, 16),           // Q8_1(h) xd*sum(q)
        16,                                          // (unused)
        32 * 16 * 4,                                 // one block of h [32][16]
        16,                                          // (unused)
        64};                                         // misc
    int fixed = 0;
    for (int v : sizes) fixed += v;
    int nst = (cap - fixed - 1024) / P.stage_bytes;
    if (nst > 16) nst = 16;
    const int scratch = al((2 * E + 64 + 2 * a.T * a.k) * 4, 16) +
                        (E + shared) * (int)sizeof(ExpertDev);   // prologue scratch in the ring
    if (nst < 2 || nst * P.stage_bytes < scratch) return cudaSuccess;
    P.nstages = nst;
    int o = nst * P.stage_bytes;
    int *offs[] = {&P.o_bar, &P.o_meta, &P.o_xq, &P.o_xd, &P.o_xs, &P.o_jobs, &P.o_stok,
                   &P.o_sw, &P.o_hq, &P.o_hd, &P.o_hs, &P.o_gu, &P.o_h, &P.o_acc, &P.o_misc};
    for (int i = 0; i < 15; i++) {
        *offs[i] = o;
        o += sizes[i];
    }
    P.smem_bytes = o;
    if (o > cap) return cudaSuccess;

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(nsm);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)P.smem_bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    err = launch_variant(cfg, P, a.T, fk, E);
    if (err != cudaSuccess) return err;
    note_launches(1);
    *taken = true;
    *look_fused = P.look.logits != nullptr;
    return cudaSuccess;
}

}  // namespace moe
