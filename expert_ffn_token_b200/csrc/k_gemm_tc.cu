// k_gemm_tc.cu -- a4-a7 for large batches on the 5th-generation tensor cores (tcgen05).
//
// Prefill on the pages runs the routed experts as grouped matrix products over the tokens that
// share an expert ("how many tokens share an expert", "Strata - the details", "Speed
// (measured)"; the MMQ-style int8 path, Strata v0.1.39 release notes).  Here each projection
// phase (gate/up, then down) is one persistent kernel, one CTA per SM, over tiles of
// (expert job, 64 tokens, 128 weight rows).
//
// Arithmetic.  A K-quant row holds, per 256-weight super-block, fp16 d and dmin and per
// 32-weight sub-block j a 6-bit scale sc_j and min m_j; the stored weight is d*sc_j*q - dmin*m_j.
// A Q8_1 activation block j of token n is xd_j[n] * qx with integer qx.  So
//   y[r][n] = sum_sb d_sb[r] * sum_{j in sb} xd_j[n] * P_j[r][n]  -  sum_j wm_j[r] * xs_j[n]
// with P_j = sum_{i in j} (sc_j * q_i) * qx_i, wm_j = RN32(dmin * m_j), xs_j = xd_j * sum qx_i.
//   * P_j is computed on the tensor cores (kind::f16): sc_j*q <= 63*31 and |qx| <= 127 are
//     integers exact in fp16, their products and 32-term sums are exact in the fp32
//     accumulator.  Every sub-block gets its own accumulator in tensor memory.
//   * the epilogue adds xd_j[n] * P_j with one FFMA per element, keeping each row's sum in
//     units of its current super-block scale (rescaled once per super-block), so that d_sb
//     costs nothing per element.
//   * the min term is a contraction over the sub-blocks, done on the tensor cores in tf32 with
//     a hi/lo split of both factors (hi*hi + hi*lo + lo*hi): relative error ~2^-22.
//   * Q8_0 rows (d_j per 32 weights, no min) rescale at every sub-block.
//   * Q5_1 rows (w = d_j*q + m_j per 32 weights) rescale at every sub-block like Q8_0 and take
//     the offsets through the min term with wm_j = -m_j (an fp16 value, exact in tf32).
// Results agree with the exact sums up to fp32 rounding.
//
// Roles (608 threads): warp 0 issues the TMA loads of the packed weights, the activation
// scales and the min-term operands, as far ahead as their rings allow; warp 18 issues the
// activation tiles into the operand stages (two producers, so that neither ring waits on the
// other); warp 1 allocates tensor memory and issues the MMAs; warps 2-9 unpack the packed
// weights into the fp16 operand (128-byte swizzled, K-major) and the per-row scales; warps
// 10-17 read the accumulators and finish the tile (SwiGLU + Q8_1(h), or the weighted scatter
// into out).  All
// hand-offs are mbarriers; every wait is bounded and a timeout ends the kernel with
// MOE_ERR_TIMEOUT.
#include <cuda.h>

#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <vector>

#include "dot.cuh"
#include "moe_internal.cuh"
#include "tc.cuh"

namespace moe {

namespace {

using namespace ptx;

constexpr int kTM = 128;           // weight rows per tile (MMA M)
constexpr int kTN = 64;            // tokens per tile (largest MMA N)
constexpr int kWSt = 2;            // 128-wide contraction stages in flight
constexpr int kRawSt = 2;          // packed super-block stages
constexpr int kMnSt = 2;           // min-term operand stages
constexpr int kEpSt = 2;           // epilogue scale stages
constexpr int kGrp = 3;            // accumulator groups: one per 64-wide stage (2 sub-blocks x 64 columns)
constexpr int kMinBuf = 2;         // min-term accumulators, one per tile
constexpr int kUnpackWarps = 8;    // two threads per weight row, one sub-block each per stage
constexpr int kEpiWarp0 = 2 + kUnpackWarps;
constexpr int kActWarp = kEpiWarp0 + 8;        // issues the activation-tile loads
constexpr int kThreads = (kActWarp + 1) * 32;
constexpr uint64_t kWaitNs = 2000000000ull;

// A 128-wide stage holds two 128-byte swizzle atoms of each operand along K:
// [A atom 0 | A atom 1 | B atom 0 | B atom 1].
constexpr uint32_t kA16 = kTM * 128;                   // one atom: 128 rows x 64 fp16
constexpr uint32_t kB16 = kTN * 128;                   // one atom: 64 tokens x 64 fp16
constexpr uint32_t kWStage = 2 * kA16 + 2 * kB16;
constexpr uint32_t kRawXd = kTN * 32;                  // 64 tokens x 8 fp32 (xd per sub-block)
constexpr uint32_t kMnWm = kTM * 32;                   // 128 rows x 8 tf32
constexpr uint32_t kMnXs = kTN * 32;                   // 64 tokens x 8 tf32
constexpr uint32_t kMnStage = 2 * kMnWm + 2 * kMnXs;
constexpr uint32_t kEpXdT = 8 * kTN * 4;               // [8][64] xd, transposed
constexpr uint32_t kEpRatio = 8 * kTM * 4;             // [8][128] unit ratios
constexpr uint32_t kEpUnit = kTM * 4;
constexpr uint32_t kEpStage = 7168;
static_assert(kEpXdT + kEpRatio + kEpUnit <= kEpStage, "epilogue stage");
constexpr int kXbPitch = 36;                           // floats per token row (bank spread)
constexpr uint32_t kXbuf = 4 * 32 * kXbPitch * 4;
constexpr int kNumBars = 2 * kWSt + 2 * kRawSt + 2 * kMnSt + 2 * kEpSt + 2 * kGrp +
                         2 * kMinBuf + 2 * 4 + 1;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kMinCol0 = kGrp * 128;              // 384

// Packed bytes of 256 weights, and how the per-row scale and the min term run for a format:
// per 32-weight block (Q8_0, Q5_1) or per super-block (K-quants); with a min/offset term
// (everything but Q8_0).
__host__ __device__ inline uint32_t sb_bytes(int fmt) {
    return fmt == MOE_FMT_Q4_K ? 144u : fmt == MOE_FMT_Q5_K ? 176u : fmt == MOE_FMT_Q8_0 ? 272u : 192u;
}
__host__ __device__ inline bool per_block_scale(int fmt) {
    return fmt == MOE_FMT_Q8_0 || fmt == MOE_FMT_Q5_1;
}
__host__ __device__ inline bool has_min(int fmt) { return fmt != MOE_FMT_Q8_0; }

struct GemmArgs {
    const CUtensorMap *wmaps;     // [n_experts (+ shared)][3] packed gate, up, down
    const ExpertDev *experts;
    const Job *jobs;
    const int32_t *njobs;
    const int32_t *perm;
    const float *w;
    int T, k, H, F, hpad;
    int K;                        // contraction length: H (gate/up) or hpad (down)
    int mt_count;                 // weight-row tiles per job
    uint32_t raw_stage;           // bytes of one packed stage (largest format present + xd)
    uint32_t raw_xd_off;          // offset of the xd tile inside a packed stage
    // gate/up outputs: Q8_1(h) as fp16 integers + scales for the down phase
    __half *hg;
    float *hgd, *hgsh, *hgsl;
    // optional exports (MOE_F_KEEP_H): fp32 h and Q8_1(h) in the int8 layout
    float *h;
    int8_t *hq;
    uint16_t *hd, *hs;
    float *hsum;
    // down outputs
    float *out;
    float *y;                     // deterministic mode: y per slot
    uint32_t *status;
};

struct Ring {
    uint32_t s = 0, ph = 0;
    __device__ __forceinline__ void adv(uint32_t depth) {
        if (++s == depth) {
            s = 0;
            ph ^= 1u;
        }
    }
};

struct Tile {
    int e, fmt, mt, slot_base, n_valid, n_mma, nbox, shared;
};

struct Cursor {
    int j = 0, base = 0;
};

// Tile i of the job-major order (job, 64-token slice, weight-row tile), tiles increasing.
__device__ __forceinline__ bool tile_at(const GemmArgs &a, int nj, Cursor &c, int i, Tile &t) {
    while (c.j < nj) {
        const Job jb = a.jobs[c.j];
        const int nt = (jb.n + kTN - 1) / kTN;
        const int cnt = nt * a.mt_count;
        if (i < c.base + cnt) {
            const int rel = i - c.base;
            const int ntile = rel / a.mt_count;
            t.mt = rel - ntile * a.mt_count;
            t.e = jb.expert;
            t.fmt = a.experts[jb.expert].fmt;
            t.slot_base = jb.slot0 + ntile * kTN;
            t.n_valid = min(kTN, jb.n - ntile * kTN);
            t.n_mma = (t.n_valid + 15) & ~15;
            t.nbox = (t.n_valid + 31) >> 5;
            t.shared = jb.shared;
            return true;
        }
        c.base += cnt;
        c.j++;
    }
    return false;
}

struct Smem {
    uint8_t *w, *raw, *mn, *ep;
    float *xb;
    uint64_t *w_full, *w_empty, *raw_full, *raw_empty, *mn_full, *mn_empty, *ep_full, *ep_empty,
        *tm_full, *tm_empty, *min_full, *min_empty, *xb_full, *xb_empty, *done;
    uint32_t *tmem_slot;
    int *abort;
};

__device__ __forceinline__ Smem carve(uint8_t *base, uint32_t raw_stage) {
    Smem s;
    uint8_t *p = base;
    s.w = p;
    p += kWSt * kWStage;
    s.raw = p;
    p += kRawSt * raw_stage;
    s.mn = p;
    p += kMnSt * kMnStage;
    s.ep = p;
    p += kEpSt * kEpStage;
    s.xb = reinterpret_cast<float *>(p);
    p += kXbuf;
    uint64_t *b = reinterpret_cast<uint64_t *>(p);
    s.w_full = b; b += kWSt;
    s.w_empty = b; b += kWSt;
    s.raw_full = b; b += kRawSt;
    s.raw_empty = b; b += kRawSt;
    s.mn_full = b; b += kMnSt;
    s.mn_empty = b; b += kMnSt;
    s.ep_full = b; b += kEpSt;
    s.ep_empty = b; b += kEpSt;
    s.tm_full = b; b += kGrp;
    s.tm_empty = b; b += kGrp;
    s.min_full = b; b += kMinBuf;
    s.min_empty = b; b += kMinBuf;
    s.xb_full = b; b += 4;
    s.xb_empty = b; b += 4;
    s.done = b; b += 1;
    s.tmem_slot = reinterpret_cast<uint32_t *>(b);
    s.abort = reinterpret_cast<int *>(b) + 1;
    return s;
}

__host__ inline size_t smem_bytes(uint32_t raw_stage) {
    return 1024 + (size_t)kWSt * kWStage + (size_t)kRawSt * raw_stage + (size_t)kMnSt * kMnStage +
           (size_t)kEpSt * kEpStage + kXbuf + (size_t)kNumBars * 8 + 16;
}

// Bounded wait on phase `parity` of `bar`; false once this CTA is aborting.
__device__ __noinline__ bool wait_bar(uint64_t *bar, uint32_t parity, int *abort,
                                      uint32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (*(volatile int *)abort) return false;
        if (globaltimer() - t0 > kWaitNs) {
            *(volatile int *)abort = 1;
            set_status(status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Fast path inline (the phase is usually complete already), bounded slow path out of line.
__device__ __forceinline__ bool wait_fast(uint64_t *bar, uint32_t parity, int *abort,
                                          uint32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar(bar, parity, abort, status);
}

// The same for all 32 lanes of a warp, with one answer for the warp.
__device__ __forceinline__ bool wait_bar_warp(uint64_t *bar, uint32_t parity, int *abort,
                                              uint32_t *status) {
    const bool ok = wait_fast(bar, parity, abort, status);
    return __all_sync(0xFFFFFFFFu, ok);
}

// silu(g) * u with the fast exponential and divide: relative error ~1e-6, far inside the
// layer's tolerance (the Q8_1 rounding of h applies to whatever h is computed).
__device__ __forceinline__ float silu_mul_fast(float g, float u) {
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ float tf32_round(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

__device__ __forceinline__ uint32_t pack_h2(int a, int b) {
    const __half2 v = __floats2half2_rn((float)a, (float)b);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ __forceinline__ float ld_half(const uint8_t *p) {
    return __half2float(*reinterpret_cast<const __half *>(p));
}

// ---------------------------------------------------------------- warps 0 and 18: TMA producers

// WHICH 0: packed weight rows + xd per super-block, and the min-term activation operands;
// WHICH 1: the fp16 activation tiles of every 128-wide operand stage.
template <int PHASE, int WHICH>
__device__ void role_producer(const GemmArgs &a, const Smem &S, int nj, const CUtensorMap *mx,
                              const CUtensorMap *md, const CUtensorMap *msh,
                              const CUtensorMap *msl) {
    Cursor cur;
    Ring rw, rr, rm;
    const int nsb = a.K / 256;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const bool mnt = has_min(t.fmt);
        const uint32_t sbb = sb_bytes(t.fmt);
        const CUtensorMap *ma, *mb;
        int ya, yb;
        if (PHASE == 0) {
            ma = a.wmaps + (size_t)t.e * 3 + 0;
            mb = a.wmaps + (size_t)t.e * 3 + 1;
            ya = yb = t.mt * 64;
        } else {
            ma = mb = a.wmaps + (size_t)t.e * 3 + 2;
            ya = t.mt * 128;
            yb = ya + 64;
        }
        for (int sb = 0; sb < nsb; sb++) {
            if (WHICH == 1) {
                for (int st = 0; st < 2; st++) {
                    if (!wait_fast(S.w_empty + rw.s, rw.ph ^ 1u, S.abort, a.status)) return;
                    uint8_t *ws = S.w + rw.s * kWStage + 2 * kA16;
                    mbar_arrive_expect_tx(S.w_full + rw.s, (uint32_t)t.nbox * 8192u);
                    for (int at = 0; at < 2; at++)
                        for (int b = 0; b < t.nbox; b++)
                            tma_load_2d(ws + at * kB16 + b * 4096, mx, (sb * 4 + 2 * st + at) * 64,
                                        t.slot_base + 32 * b, S.w_full + rw.s);
                    rw.adv(kWSt);
                }
                continue;
            }
            if (!wait_fast(S.raw_empty + rr.s, rr.ph ^ 1u, S.abort, a.status)) return;
            uint8_t *rs = S.raw + rr.s * a.raw_stage;
            mbar_arrive_expect_tx(S.raw_full + rr.s, 128u * sbb + (uint32_t)t.nbox * 1024u);
            // Q8_0 maps count 16-bit elements (34-byte blocks), the others bytes
            const int x = t.fmt == MOE_FMT_Q8_0 ? sb * 136 : sb * (int)sbb;
            tma_load_2d(rs, ma, x, ya, S.raw_full + rr.s);
            tma_load_2d(rs + 64 * sbb, mb, x, yb, S.raw_full + rr.s);
            for (int b = 0; b < t.nbox; b++)
                tma_load_2d(rs + a.raw_xd_off + b * 1024, md, sb * 8, t.slot_base + 32 * b,
                            S.raw_full + rr.s);
            rr.adv(kRawSt);
            if (mnt) {
                if (!wait_fast(S.mn_empty + rm.s, rm.ph ^ 1u, S.abort, a.status)) return;
                uint8_t *ms = S.mn + rm.s * kMnStage;
                mbar_arrive_expect_tx(S.mn_full + rm.s, (uint32_t)t.nbox * 2048u);
                for (int b = 0; b < t.nbox; b++) {
                    tma_load_2d(ms + 2 * kMnWm + b * 1024, msh, sb * 8, t.slot_base + 32 * b,
                                S.mn_full + rm.s);
                    tma_load_2d(ms + 2 * kMnWm + kMnXs + b * 1024, msl, sb * 8,
                                t.slot_base + 32 * b, S.mn_full + rm.s);
                }
                rm.adv(kMnSt);
            }
        }
    }
}

// ---------------------------------------------------------------- warps 2-9: unpack

// Operand order along K.  Inside every group of 4 consecutive weights the operands hold the
// elements in the order (0, 2, 1, 3); both sides use the same order, so the products and sums
// are unchanged.  This lets two 4-bit fields of one 32-bit word become an fp16 pair with one
// lop3 (0x6400 | q is the fp16 value 1024 + q).
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t x, uint32_t m, uint32_t c) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(m), "r"(c));   // (x & m) | c
    return r;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}
__device__ __forceinline__ uint32_t hfma2_u(uint32_t a, uint32_t b, uint32_t c) {
    const __half2 r = __hfma2(*reinterpret_cast<const __half2 *>(&a),
                              *reinterpret_cast<const __half2 *>(&b),
                              *reinterpret_cast<const __half2 *>(&c));
    return *reinterpret_cast<const uint32_t *>(&r);
}
__device__ __forceinline__ uint32_t hsub2_u(uint32_t a, uint32_t b) {
    const __half2 r = __hsub2(*reinterpret_cast<const __half2 *>(&a),
                              *reinterpret_cast<const __half2 *>(&b));
    return *reinterpret_cast<const uint32_t *>(&r);
}
// fp16 pair (s, s) and (-1024 s, -1024 s): fma(1024 + q, s, -1024 s) = q * s exactly, for
// integers q <= 31 and s <= 63 (the product is exact in fp16 and the fma rounds once).
__device__ __forceinline__ void scale_pair(int s, uint32_t &s2, uint32_t &nb2) {
    const __half2 a = __float2half2_rn((float)s);
    const __half2 b = __float2half2_rn(-1024.0f * (float)s);
    s2 = *reinterpret_cast<const uint32_t *>(&a);
    nb2 = *reinterpret_cast<const uint32_t *>(&b);
}

// Row r's 32 weights of sub-block j = 2 st + hsel as fp16 integers sc_j * q (K-quants) or q
// (Q8_0, Q5_1), written into their half of the 128-byte-swizzled K-major operand row.
template <int FMT>
__device__ __forceinline__ void unpack_half(const uint8_t *rowp, int st, int hsel, int scale,
                                            bool zero, uint8_t *a16, int r) {
    constexpr uint32_t kM = 0x000F000Fu, kE = 0x64006400u;
    uint32_t v[16];
    if (FMT == MOE_FMT_Q8_0) {
        // bytes b -> fp16 (1024 + (b ^ 0x80)) - 1152 = b
        const uint32_t k1152 = 0x64806480u;
        const uint8_t *blk = rowp + 34 * (2 * st + hsel);
        const uint16_t d16 = *reinterpret_cast<const uint16_t *>(blk);
        const bool z = zero || d16 == 0 || d16 == 0x8000u;
        const uint16_t *qp = reinterpret_cast<const uint16_t *>(blk + 2);
#pragma unroll
        for (int wi = 0; wi < 8; wi++) {
            const uint32_t x =
                ((uint32_t)qp[2 * wi] | ((uint32_t)qp[2 * wi + 1] << 16)) ^ 0x80808080u;
            const uint32_t a = hsub2_u(prmt(x, 0x64646464u, 0x4240u), k1152);
            const uint32_t b = hsub2_u(prmt(x, 0x64646464u, 0x4341u), k1152);
            v[2 * wi] = z ? 0u : a;
            v[2 * wi + 1] = z ? 0u : b;
        }
    } else if (FMT == MOE_FMT_Q5_1) {
        // element n < 16: low nibble of qs[n], n >= 16: high nibble of qs[n - 16]; bit n of qh
        // is its fifth bit.  Word wi of the operand covers elements 4 wi .. 4 wi + 3.
        const uint2 *bp = reinterpret_cast<const uint2 *>(rowp + 24 * (2 * st + hsel));
        const uint2 h = bp[0], qa = bp[1], qb = bp[2];
        const bool z = zero || (h.x & 0x7FFFu) == 0;
        const uint32_t qw[4] = {qa.x, qa.y, qb.x, qb.y};
#pragma unroll
        for (int wi = 0; wi < 8; wi++) {
            const uint32_t x = wi < 4 ? qw[wi] : qw[wi - 4] >> 4;
            const uint32_t t = h.y >> (4 * wi);
            // bits 0, 2 of t -> bits 4, 20 (elements k, k+2); bits 1, 3 -> (k+1, k+3)
            const uint32_t a = lop3_and_or(x, kM, kE) | (((t & 5u) * 0x40010u) & 0x00100010u);
            const uint32_t b = lop3_and_or(x >> 8, kM, kE) | (((t & 10u) * 0x20008u) & 0x00100010u);
            v[2 * wi] = z ? 0u : hsub2_u(a, kE);
            v[2 * wi + 1] = z ? 0u : hsub2_u(b, kE);
        }
    } else {
        const int qs_off = FMT == MOE_FMT_Q5_K ? 48 : 16;
        const uint4 *qp = reinterpret_cast<const uint4 *>(rowp + qs_off + 32 * st);
        const uint4 qa = qp[0], qb = qp[1];
        const uint32_t qw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
        uint32_t hw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (FMT == MOE_FMT_Q5_K) {
            const uint4 *hp = reinterpret_cast<const uint4 *>(rowp + 16);
            const uint4 ha = hp[0], hb2 = hp[1];
            hw[0] = ha.x; hw[1] = ha.y; hw[2] = ha.z; hw[3] = ha.w;
            hw[4] = hb2.x; hw[5] = hb2.y; hw[6] = hb2.z; hw[7] = hb2.w;
        }
        const int j = 2 * st + hsel, sh = 4 * hsel;   // low nibbles: sub-block 2st, high: 2st+1
        uint32_t s2, n2;
        scale_pair(zero ? 0 : scale, s2, n2);
#pragma unroll
        for (int wi = 0; wi < 8; wi++) {
            const uint32_t x = qw[wi] >> sh;
            uint32_t a = lop3_and_or(x, kM, kE);          // elements k, k+2
            uint32_t b = lop3_and_or(x >> 8, kM, kE);     // k+1, k+3
            if (FMT == MOE_FMT_Q5_K) {                    // fifth bit -> value bit 4
                const uint32_t t = hw[wi] >> j;
                a |= (t << 4) & 0x00100010u;
                b |= (t >> 4) & 0x00100010u;
            }
            v[2 * wi] = hfma2_u(a, s2, n2);
            v[2 * wi + 1] = hfma2_u(b, s2, n2);
        }
    }
    uint8_t *rowbase = a16 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
    for (int c = 0; c < 4; c++) {
        *reinterpret_cast<uint4 *>(rowbase + (((4 * hsel + c) ^ (r & 7)) << 4)) =
            make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    }
}

template <int FMT>
__device__ __forceinline__ bool unpack_superblock(const GemmArgs &a, const Smem &S, Ring &rw,
                                                  Ring &rm, Ring &re, const uint8_t *rs,
                                                  float &U, int u) {
    const int r = u >> 1, hsel = u & 1;        // weight row, sub-block within each stage
    const int lane = threadIdx.x & 31;
    const uint32_t sbb = sb_bytes(FMT);
    const uint8_t *rowp = rs + (size_t)r * sbb;
    int sc[8], mn[8];
    float d = 0.f, dmin = 0.f;
    float off[8];                              // Q5_1: the blocks' offsets m_j
    // ---- epilogue scales: unit ratios, unit, transposed xd
    if (!wait_bar_warp(S.ep_empty + re.s, re.ph ^ 1u, S.abort, a.status)) return false;
    uint8_t *es = S.ep + re.s * kEpStage;
    float *xdT = reinterpret_cast<float *>(es);
    float *ratio = reinterpret_cast<float *>(es + kEpXdT);
    float *unit = reinterpret_cast<float *>(es + kEpXdT + kEpRatio);
    if (!per_block_scale(FMT)) {
        d = ld_half(rowp);
        dmin = ld_half(rowp + 2);
        const uint32_t s0 = *reinterpret_cast<const uint32_t *>(rowp + 4);
        const uint32_t s1 = *reinterpret_cast<const uint32_t *>(rowp + 8);
        const uint32_t s2 = *reinterpret_cast<const uint32_t *>(rowp + 12);
#pragma unroll
        for (int j = 0; j < 8; j++) kq_scale_min(s0, s1, s2, j, sc[j], mn[j]);
        float rt = 1.0f;
        if (d != 0.0f) {
            rt = __fdiv_rn(U, d);
            U = d;
        }
        if (hsel == 0) ratio[r] = rt;
    } else {
        constexpr int kBB = FMT == MOE_FMT_Q8_0 ? 34 : 24;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            sc[j] = 1;
            mn[j] = 0;
            off[j] = FMT == MOE_FMT_Q5_1 ? ld_half(rowp + kBB * j + 2) : 0.0f;
            const float dj = ld_half(rowp + kBB * j);
            float rt = 1.0f;
            if (dj != 0.0f) {
                rt = __fdiv_rn(U, dj);
                U = dj;
            }
            if (hsel == 0) ratio[j * kTM + r] = rt;
        }
    }
    if (hsel == 0) unit[r] = U;
    if (u < kTN) {
        const float4 *src = reinterpret_cast<const float4 *>(rs + a.raw_xd_off + u * 32);
        const float4 x0 = src[0], x1 = src[1];
        xdT[0 * kTN + u] = x0.x;
        xdT[1 * kTN + u] = x0.y;
        xdT[2 * kTN + u] = x0.z;
        xdT[3 * kTN + u] = x0.w;
        xdT[4 * kTN + u] = x1.x;
        xdT[5 * kTN + u] = x1.y;
        xdT[6 * kTN + u] = x1.z;
        xdT[7 * kTN + u] = x1.w;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(S.ep_full + re.s);
    re.adv(kEpSt);
    // ---- min-term operand rows: RN32(dmin * m_j) (K-quants) or -m_j (Q5_1), split into
    // tf32 hi + lo (for Q5_1 lo is 0: an fp16 value is exact in tf32)
    if (has_min(FMT)) {
        if (!wait_bar_warp(S.mn_empty + rm.s, rm.ph ^ 1u, S.abort, a.status)) return false;
        uint8_t *ms = S.mn + rm.s * kMnStage;
        float wh[8], wl[8];
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const float wm = FMT == MOE_FMT_Q5_1 ? -off[j] : __fmul_rn(dmin, (float)mn[j]);
            wh[j] = tf32_round(wm);
            wl[j] = wm - wh[j];
        }
        const int sw = (r >> 2) & 1;
        if (hsel == 0) {
            float4 *dh = reinterpret_cast<float4 *>(ms + r * 32);
            dh[0 ^ sw] = make_float4(wh[0], wh[1], wh[2], wh[3]);
            dh[1 ^ sw] = make_float4(wh[4], wh[5], wh[6], wh[7]);
        } else {
            float4 *dl = reinterpret_cast<float4 *>(ms + kMnWm + r * 32);
            dl[0 ^ sw] = make_float4(wl[0], wl[1], wl[2], wl[3]);
            dl[1 ^ sw] = make_float4(wl[4], wl[5], wl[6], wl[7]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(S.mn_full + rm.s);
        rm.adv(kMnSt);
    }
    // ---- the two 128-wide operand stages (two swizzle atoms, four sub-blocks each)
    const bool zero = !per_block_scale(FMT) && d == 0.0f;
    for (int st = 0; st < 2; st++) {
        if (!wait_bar_warp(S.w_empty + rw.s, rw.ph ^ 1u, S.abort, a.status)) return false;
        uint8_t *a16 = S.w + rw.s * kWStage;
        unpack_half<FMT>(rowp, 2 * st, hsel, sc[4 * st + hsel], zero, a16, r);
        unpack_half<FMT>(rowp, 2 * st + 1, hsel, sc[4 * st + 2 + hsel], zero, a16 + kA16, r);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(S.w_full + rw.s);
        rw.adv(kWSt);
    }
    return true;
}

template <int PHASE>
__device__ void role_unpack(const GemmArgs &a, const Smem &S, int nj) {
    const int u = threadIdx.x - 64;              // 0..255: row u / 2, sub-block u % 2
    const int lane = threadIdx.x & 31;
    Cursor cur;
    Ring rw, rr, rm, re;
    const int nsb = a.K / 256;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        float U = 1.0f;
        for (int sb = 0; sb < nsb; sb++) {
            if (!wait_bar_warp(S.raw_full + rr.s, rr.ph, S.abort, a.status)) return;
            const uint8_t *rs = S.raw + rr.s * a.raw_stage;
            bool ok;
            if (t.fmt == MOE_FMT_Q4_K)
                ok = unpack_superblock<MOE_FMT_Q4_K>(a, S, rw, rm, re, rs, U, u);
            else if (t.fmt == MOE_FMT_Q5_K)
                ok = unpack_superblock<MOE_FMT_Q5_K>(a, S, rw, rm, re, rs, U, u);
            else if (t.fmt == MOE_FMT_Q8_0)
                ok = unpack_superblock<MOE_FMT_Q8_0>(a, S, rw, rm, re, rs, U, u);
            else
                ok = unpack_superblock<MOE_FMT_Q5_1>(a, S, rw, rm, re, rs, U, u);
            if (!ok) return;
            __syncwarp();
            if (lane == 0) mbar_arrive(S.raw_empty + rr.s);
            rr.adv(kRawSt);
        }
    }
}

// ---------------------------------------------------------------- warp 1: MMA issuer

template <int PHASE>
__device__ void role_mma(const GemmArgs &a, const Smem &S, int nj, uint32_t tbase) {
    Cursor cur;
    Ring rw, rm, rj, rmin;
    const int nsb = a.K / 256;
    // Descriptors of stage 0; stage s and sub-block offsets are added to the start-address field
    // (16-byte units; no carry out of the field since shared addresses stay below 256 KB).
    const uint64_t dA0 = smem_desc(smem_u32(S.w), 1024, 2);
    const uint64_t dB0 = smem_desc(smem_u32(S.w) + 2 * kA16, 1024, 2);
    const uint64_t dM0 = smem_desc(smem_u32(S.mn), 256, 6);
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const bool mnt = has_min(t.fmt);
        const uint32_t idf = instr_desc(0, kTM, t.n_mma);
        const uint32_t idt = instr_desc(2, kTM, t.n_mma);
        for (int sb = 0; sb < nsb; sb++) {
            for (int st = 0; st < 2; st++) {
                // one 128-wide stage = two swizzle atoms; each atom holds two sub-blocks, each
                // into its own 64-column accumulator of one group
                if (!wait_fast(S.w_full + rw.s, rw.ph, S.abort, a.status)) return;
                const uint64_t so = (uint64_t)(rw.s * (kWStage >> 4));
#pragma unroll
                for (int at = 0; at < 2; at++) {
                    if (!wait_fast(S.tm_empty + rj.s, rj.ph ^ 1u, S.abort, a.status)) return;
                    tc_fence_after();
                    const uint64_t da = dA0 + so + at * (kA16 >> 4), db = dB0 + so + at * (kB16 >> 4);
                    const uint32_t d0 = tbase + rj.s * 128;
                    umma_f16(d0, da, db, idf, 0u);
                    umma_f16(d0, da + 2, db + 2, idf, 1u);
                    umma_f16(d0 + 64, da + 4, db + 4, idf, 0u);
                    umma_f16(d0 + 64, da + 6, db + 6, idf, 1u);
                    umma_commit(S.tm_full + rj.s);
                    rj.adv(kGrp);
                }
                umma_commit(S.w_empty + rw.s);
                rw.adv(kWSt);
            }
            if (mnt) {
                if (!wait_fast(S.mn_full + rm.s, rm.ph, S.abort, a.status)) return;
                if (sb == 0 && !wait_fast(S.min_empty + rmin.s, rmin.ph ^ 1u, S.abort, a.status))
                    return;
                tc_fence_after();
                const uint64_t mo = (uint64_t)(rm.s * (kMnStage >> 4));
                const uint64_t wh = dM0 + mo, wl = wh + (kMnWm >> 4), xh = wh + (2 * kMnWm >> 4),
                               xl = xh + (kMnXs >> 4);
                const uint32_t dm = tbase + kMinCol0 + rmin.s * 64;
                umma_tf32(dm, wh, xh, idt, sb > 0 ? 1u : 0u);
                umma_tf32(dm, wh, xl, idt, 1u);
                umma_tf32(dm, wl, xh, idt, 1u);
                umma_commit(S.mn_empty + rm.s);
                rm.adv(kMnSt);
            }
        }
        if (mnt) {
            umma_commit(S.min_full + rmin.s);
            rmin.adv(kMinBuf);
        }
    }
}

// ---------------------------------------------------------------- warps 10-17: epilogue

// Q8_1 of 32 consecutive h values of one token (the reading of the quantizer the rest of the
// library uses), stored as fp16 integers + scales for the down phase, and optionally in the
// exported int8 layout.
__device__ __noinline__ void quantize_h_block(const GemmArgs &a, const float *v32, int slot,
                                                 int f0) {
    float v[32];
#pragma unroll
    for (int c = 0; c < 8; c++) {
        const float4 x = reinterpret_cast<const float4 *>(v32)[c];
        v[4 * c] = x.x;
        v[4 * c + 1] = x.y;
        v[4 * c + 2] = x.z;
        v[4 * c + 3] = x.w;
    }
    bool fin = true;
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 32; i++) {
        fin = fin && isfinite(v[i]);
        am = fmaxf(am, fabsf(v[i]));
    }
    const float d = __fdiv_rn(am, 127.0f);
    int q[32];
    int sum = 0;
    if (fin && d != 0.0f) {
        // q = round-half-away(RN(v / d)).  For normal d, v * RN(1/d) is within 2 ulp of
        // RN(v / d), and |v / d| <= 127 makes 2 ulp < 2^-15: unless the product lies that close
        // to a half-integer, both round to the same integer.  The rare close cases, and a
        // subnormal d, take the IEEE division.
        const bool fast = d >= 0x1p-125f;
        const float inv = __frcp_rn(d);
#pragma unroll
        for (int i = 0; i < 32; i++) {
            const float r = v[i] * inv;
            const float a = fabsf(r);
            const bool near_tie = !fast || fabsf(a - floorf(a) - 0.5f) < 0x1p-15f;
            const float rq = near_tie ? __fdiv_rn(v[i], d) : r;
            const int qi = max(-127, min(127, (int)roundf(rq)));
            q[i] = qi;
            sum += qi;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; i++) q[i] = 0;
    }
    const int hb = a.hpad / 32;
    const size_t bi = (size_t)slot * hb + f0 / 32;
    const __half dh = __float2half_rn(d);
    const float dhf = fin ? __half2float(dh) : 0.0f;
    const float xs = fin ? __fmul_rn(__half2float(dh), (float)sum) : 0.0f;
    uint4 *dst = reinterpret_cast<uint4 *>(a.hg + (size_t)slot * a.hpad + f0);
#pragma unroll
    for (int c = 0; c < 4; c++)     // operand order (0, 2, 1, 3) inside every 4
        dst[c] = make_uint4(pack_h2(q[8 * c], q[8 * c + 2]), pack_h2(q[8 * c + 1], q[8 * c + 3]),
                            pack_h2(q[8 * c + 4], q[8 * c + 6]),
                            pack_h2(q[8 * c + 5], q[8 * c + 7]));
    a.hgd[bi] = dhf;
    const float xh = tf32_round(xs);
    a.hgsh[bi] = xh;
    a.hgsl[bi] = tf32_round(xs - xh);
    if (a.hq) {
        uint32_t qb[8];
#pragma unroll
        for (int c = 0; c < 8; c++)
            qb[c] = (uint32_t)(q[4 * c] & 0xFF) | ((uint32_t)(q[4 * c + 1] & 0xFF) << 8) |
                    ((uint32_t)(q[4 * c + 2] & 0xFF) << 16) |
                    ((uint32_t)(q[4 * c + 3] & 0xFF) << 24);
        uint4 *hqd = reinterpret_cast<uint4 *>(a.hq + (size_t)slot * a.hpad + f0);
        hqd[0] = make_uint4(qb[0], qb[1], qb[2], qb[3]);
        hqd[1] = make_uint4(qb[4], qb[5], qb[6], qb[7]);
        a.hd[bi] = fin ? __half_as_ushort(dh) : 0;
        a.hs[bi] = fin ? __half_as_ushort(__float2half_rn(__fmul_rn(d, (float)sum))) : 0;
        a.hsum[bi] = xs;
        float4 *hf = reinterpret_cast<float4 *>(a.h + (size_t)slot * a.F + f0);
#pragma unroll
        for (int c = 0; c < 8; c++)
            hf[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    }
    if (!fin) set_status(a.status, MOE_ERR_NONFINITE);
}

template <int PHASE>
__device__ void role_epilogue(const GemmArgs &a, const Smem &S, int nj, uint32_t tbase) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;                  // tensor-memory lane quarter of this warp
    const int hcol = (warp - kEpiWarp0) >> 2;  // column half: tokens [32 hcol, 32 hcol + 32)
    const int r = 32 * q + lane;             // weight row of the tile
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    Cursor cur;
    Ring re, rj, rmin, rx;
    const int nsb = a.K / 256;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const bool pbs = per_block_scale(t.fmt), mnt = has_min(t.fmt);
        const int ncol = min(32, t.n_valid - 32 * hcol);
        const bool active = ncol > 0;
        float acc[32];
#pragma unroll
        for (int c = 0; c < 32; c++) acc[c] = 0.f;
        float U = 1.0f;
        uint32_t P[16];
        const int nst_tile = nsb * 4;
        const float *xdT = nullptr, *ratio = nullptr, *unit = nullptr;
        for (int sg = 0; sg < nst_tile; sg++) {
            const int st = sg & 3;
            if (st == 0) {
                if (!wait_bar_warp(S.ep_full + re.s, re.ph, S.abort, a.status)) return;
                const uint8_t *es = S.ep + re.s * kEpStage;
                xdT = reinterpret_cast<const float *>(es);
                ratio = reinterpret_cast<const float *>(es + kEpXdT);
                unit = reinterpret_cast<const float *>(es + kEpXdT + kEpRatio);
                if (!pbs && active) {
                    const float rt = ratio[r];
#pragma unroll
                    for (int c = 0; c < 32; c++) acc[c] *= rt;
                }
            }
            if (!wait_bar_warp(S.tm_full + rj.s, rj.ph, S.abort, a.status)) return;
            tc_fence_after();
            if (active) {
                const uint32_t ta = tbase + lane_addr + rj.s * 128 + 32 * hcol;
#pragma unroll 1
                for (int h2 = 0; h2 < 2; h2++) {
                    const int jj = 2 * st + h2;
                    if (pbs) {
                        const float rt = ratio[jj * kTM + r];
#pragma unroll
                        for (int c = 0; c < 32; c++) acc[c] *= rt;
                    }
#pragma unroll
                    for (int q16 = 0; q16 < 2; q16++) {
                        tmem_ld16(ta + 64 * h2 + 16 * q16, P);
                        tmem_ld_wait(P);
                        const float4 *xd4 =
                            reinterpret_cast<const float4 *>(xdT + jj * kTN + 32 * hcol + 16 * q16);
#pragma unroll
                        for (int c4 = 0; c4 < 4; c4++) {
                            const float4 x = xd4[c4];
                            float *ac = acc + 16 * q16 + 4 * c4;
                            ac[0] = fmaf(__uint_as_float(P[4 * c4 + 0]), x.x, ac[0]);
                            ac[1] = fmaf(__uint_as_float(P[4 * c4 + 1]), x.y, ac[1]);
                            ac[2] = fmaf(__uint_as_float(P[4 * c4 + 2]), x.z, ac[2]);
                            ac[3] = fmaf(__uint_as_float(P[4 * c4 + 3]), x.w, ac[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(S.tm_empty + rj.s);
            rj.adv(kGrp);
            if (st == 3) {
                U = unit[r];
                __syncwarp();
                if (lane == 0) mbar_arrive(S.ep_empty + re.s);
                re.adv(kEpSt);
            }
        }
        // min term, then the row scale: y = acc * U - min
#pragma unroll
        for (int c = 0; c < 32; c++) acc[c] *= U;
        if (mnt) {
            if (!wait_bar_warp(S.min_full + rmin.s, rmin.ph, S.abort, a.status)) return;
            tc_fence_after();
            if (active) {
#pragma unroll
                for (int q16 = 0; q16 < 2; q16++) {
                    tmem_ld16(tbase + lane_addr + kMinCol0 + rmin.s * 64 + 32 * hcol + 16 * q16, P);
                    tmem_ld_wait(P);
#pragma unroll
                    for (int c = 0; c < 16; c++) acc[16 * q16 + c] -= __uint_as_float(P[c]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(S.min_empty + rmin.s);
            rmin.adv(kMinBuf);
        }
        if (!active) continue;

        if (PHASE == 0) {
            // rows 0..63 are gate rows m0..m0+63, rows 64..127 the up rows of the same f
            // the up warp hands its 32 x 32 block to the gate warp of the same rows and tokens
            const int p = q & 1;
            const bool is_up = q >= 2;
            const int pi = p * 2 + hcol;
            float *xb = S.xb + pi * 32 * kXbPitch;
            if (is_up) {
                if (!wait_bar_warp(S.xb_empty + pi, rx.ph ^ 1u, S.abort, a.status)) return;
#pragma unroll
                for (int c = 0; c < 32; c++) xb[c * kXbPitch + lane] = acc[c];
                __syncwarp();
                if (lane == 0) mbar_arrive(S.xb_full + pi);
            } else {
                if (!wait_bar_warp(S.xb_full + pi, rx.ph, S.abort, a.status)) return;
#pragma unroll
                for (int c = 0; c < 32; c++)
                    xb[c * kXbPitch + lane] = silu_mul_fast(acc[c], xb[c * kXbPitch + lane]);
                __syncwarp();
                const int f0 = t.mt * 64 + 32 * p;
                if (lane < ncol && f0 < a.F)
                    quantize_h_block(a, xb + lane * kXbPitch, t.slot_base + 32 * hcol + lane, f0);
                __syncwarp();
                if (lane == 0) mbar_arrive(S.xb_empty + pi);
            }
            rx.adv(1);
        } else {
            const int slot_c = t.slot_base + 32 * hcol + lane;
            int tok = 0;
            float wt = 0.f;
            if (lane < ncol) {
                if (t.shared) {
                    tok = slot_c - a.T * a.k;
                    wt = 1.0f;
                } else {
                    const int pp = a.perm[slot_c];
                    tok = pp / a.k;
                    wt = a.w[pp];
                }
            }
            const int i_row = t.mt * kTM + r;
#pragma unroll
            for (int c = 0; c < 32; c++) {
                const int tc = __shfl_sync(0xFFFFFFFFu, tok, c);
                const float wc = __shfl_sync(0xFFFFFFFFu, wt, c);
                if (c < ncol && i_row < a.H) {
                    if (a.y)
                        a.y[(size_t)(t.slot_base + 32 * hcol + c) * a.H + i_row] = acc[c];
                    else
                        atomicAdd(a.out + (size_t)tc * a.H + i_row, wc * acc[c]);
                }
            }
        }
    }
}

// ---------------------------------------------------------------- the kernel

template <int PHASE>
__global__ void __maxnreg__(96)
    k_gemm_tc(const GemmArgs a, const __grid_constant__ CUtensorMap map_x,
              const __grid_constant__ CUtensorMap map_d,
              const __grid_constant__ CUtensorMap map_sh,
              const __grid_constant__ CUtensorMap map_sl) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const Smem S = carve(base, a.raw_stage);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kWSt; i++) {
            mbar_init(S.w_full + i, 1 + kUnpackWarps);
            mbar_init(S.w_empty + i, 1);
        }
        for (int i = 0; i < kRawSt; i++) {
            mbar_init(S.raw_full + i, 1);
            mbar_init(S.raw_empty + i, kUnpackWarps);
        }
        for (int i = 0; i < kMnSt; i++) {
            mbar_init(S.mn_full + i, 1 + kUnpackWarps);
            mbar_init(S.mn_empty + i, 1);
        }
        for (int i = 0; i < kEpSt; i++) {
            mbar_init(S.ep_full + i, kUnpackWarps);
            mbar_init(S.ep_empty + i, 8);
        }
        for (int i = 0; i < kGrp; i++) {
            mbar_init(S.tm_full + i, 1);
            mbar_init(S.tm_empty + i, 8);
        }
        for (int i = 0; i < kMinBuf; i++) {
            mbar_init(S.min_full + i, 1);
            mbar_init(S.min_empty + i, 8);
        }
        for (int i = 0; i < 4; i++) {
            mbar_init(S.xb_full + i, 1);
            mbar_init(S.xb_empty + i, 1);
        }
        mbar_init(S.done, 1);
        *S.abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(S.tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *S.tmem_slot;
    const int nj = *a.njobs;

    if (warp == 0) {
        if (lane == 0) role_producer<PHASE, 0>(a, S, nj, &map_x, &map_d, &map_sh, &map_sl);
        __syncwarp();
    } else if (warp == kActWarp) {
        if (lane == 0) role_producer<PHASE, 1>(a, S, nj, &map_x, &map_d, &map_sh, &map_sl);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            role_mma<PHASE>(a, S, nj, tbase);
            umma_commit(S.done);
            wait_bar(S.done, 0, S.abort, a.status);
        }
        __syncwarp();
    } else if (warp < kEpiWarp0) {
        role_unpack<PHASE>(a, S, nj);
        __syncwarp();
    } else {
        role_epilogue<PHASE>(a, S, nj, tbase);
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (*(volatile int *)S.abort) {
        // copies already issued land before the CTA leaves
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 200000ull) {
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// ---------------------------------------------------------------- gather + tail kernels

// Slot-ordered activation operand for the gate/up phase: the Q8_1 integers of each slot's
// token as fp16, xd per block as fp32, and xsum split into tf32 hi + lo.  One warp per slot.
__global__ void __launch_bounds__(256) k_act_gather(const int8_t *__restrict__ xq,
                                                    const uint16_t *__restrict__ xd,
                                                    const float *__restrict__ xsum,
                                                    const int32_t *__restrict__ perm, int T, int k,
                                                    int H, int slots, __half *xg, float *xgd,
                                                    float *xgsh, float *xgsl) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= slots) return;
    const int s = warp;
    const int t = s < T * k ? perm[s] / k : s - T * k;
    const int8_t *src = xq + (size_t)t * H;
    __half *dst = xg + (size_t)s * H;
    for (int c = lane; c < H / 8; c += 32) {
        const uint2 v = *reinterpret_cast<const uint2 *>(src + 8 * c);
        const int8_t *b = reinterpret_cast<const int8_t *>(&v);
        uint4 o;                    // operand order (0, 2, 1, 3) inside every 4
        o.x = pack_h2(b[0], b[2]);
        o.y = pack_h2(b[1], b[3]);
        o.z = pack_h2(b[4], b[6]);
        o.w = pack_h2(b[5], b[7]);
        *reinterpret_cast<uint4 *>(dst + 8 * c) = o;
    }
    const int nb = H / 32;
    for (int j = lane; j < nb; j += 32) {
        const size_t si = (size_t)t * nb + j, di = (size_t)s * nb + j;
        xgd[di] = half_bits_to_float(xd[si]);
        const float xs = xsum[si];
        const float hi = tf32_round(xs);
        xgsh[di] = hi;
        xgsl[di] = tf32_round(xs - hi);
    }
}

// Zero the fp16 h operand and its scales in the padded columns [F, hpad) of every slot.
__global__ void k_hg_tail_zero(__half *hg, float *hgd, float *hgsh, float *hgsl, int slots, int F,
                               int hpad) {
    const int nbt = (hpad - F) / 32;
    const int hb = hpad / 32;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < slots * nbt;
         i += gridDim.x * blockDim.x) {
        const int s = i / nbt, b = F / 32 + i % nbt;
        uint4 *p = reinterpret_cast<uint4 *>(hg + (size_t)s * hpad + b * 32);
#pragma unroll
        for (int c = 0; c < 4; c++) p[c] = make_uint4(0, 0, 0, 0);
        hgd[(size_t)s * hb + b] = 0.f;
        hgsh[(size_t)s * hb + b] = 0.f;
        hgsl[(size_t)s * hb + b] = 0.f;
    }
}

// ---------------------------------------------------------------- host side

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    static std::once_flag once;
    static EncodeFn fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    });
    return fn;
}

bool encode_2d(CUtensorMap *m, CUtensorMapDataType dt, size_t esize, const void *base,
               uint64_t dim0, uint64_t dim1, uint64_t stride_bytes, uint32_t box0, uint32_t box1,
               CUtensorMapSwizzle sw) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    (void)esize;
    const cuuint64_t dims[2] = {dim0, dim1};
    const cuuint64_t strides[1] = {stride_bytes};
    const cuuint32_t box[2] = {box0, box1};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
    static std::mutex mu;
    static std::vector<int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
    if (!cache[dev]) cudaDeviceGetAttribute(&cache[dev], cudaDevAttrMultiProcessorCount, dev);
    return cache[dev];
}

}  // namespace

// Tensor maps of every expert's three packed matrices, as boxes of one super-block (256
// weights) x 64 rows.  Returns false when a map cannot be encoded (the caller then keeps the
// CUDA-core kernels for large batches).
bool tc_build_weight_maps(const uint8_t *d_base, const moe_expert_desc *descs, int n, int H,
                          int F, std::vector<uint8_t> &out) {
    if (H % 256 != 0) return false;
    out.assign((size_t)n * 3 * sizeof(CUtensorMap), 0);
    CUtensorMap *maps = reinterpret_cast<CUtensorMap *>(out.data());
    for (int e = 0; e < n; e++) {
        const moe_expert_desc &d = descs[e];
        for (int t = 0; t < 3; t++) {
            const int rows = t < 2 ? F : H;
            const int width = t < 2 ? H : F;
            const void *base = d_base + d.off[t];
            bool ok;
            if (d.fmt == MOE_FMT_Q8_0) {
                const uint64_t nb = (uint64_t)((width + 31) / 32);
                ok = encode_2d(&maps[e * 3 + t], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, base, nb * 17,
                               (uint64_t)rows, d.stride[t], 136, 64, CU_TENSOR_MAP_SWIZZLE_NONE);
            } else if (d.fmt == MOE_FMT_Q5_1) {
                const uint64_t nb = (uint64_t)((width + 31) / 32);
                ok = encode_2d(&maps[e * 3 + t], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, nb * 24,
                               (uint64_t)rows, d.stride[t], 192, 64, CU_TENSOR_MAP_SWIZZLE_NONE);
            } else {
                const uint32_t sbb = sb_bytes(d.fmt);
                const uint64_t nsb = (uint64_t)((width + 255) / 256);
                ok = encode_2d(&maps[e * 3 + t], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, nsb * sbb,
                               (uint64_t)rows, d.stride[t], sbb, 64, CU_TENSOR_MAP_SWIZZLE_NONE);
            }
            if (!ok) return false;
        }
    }
    return true;
}

size_t tc_map_bytes() { return sizeof(CUtensorMap); }

// One projection phase on the tensor cores.  phase 0: gate/up (K = H) writing Q8_1(h);
// phase 1: down (K = hpad) writing out (or y per slot).
cudaError_t launch_gemm_tc(const TcPhaseArgs &p, cudaStream_t st) {
    const FfnArgs &f = p.ffn;
    GemmArgs a{};
    a.wmaps = reinterpret_cast<const CUtensorMap *>(p.wmaps);
    a.experts = f.experts;
    a.jobs = f.jobs;
    a.njobs = f.njobs;
    a.perm = f.perm;
    a.w = f.w;
    a.T = f.T;
    a.k = f.k;
    a.H = f.H;
    a.F = f.F;
    a.hpad = f.hpad;
    a.K = p.phase == 0 ? f.H : f.hpad;
    a.mt_count = p.phase == 0 ? (f.F + 63) / 64 : (f.H + kTM - 1) / kTM;
    uint32_t sbb_max = 0;
    for (int fm = 0; fm <= MOE_FMT_Q5_1; fm++)
        if (f.fmt_mask & (1 << fm)) sbb_max = sbb_max > sb_bytes(fm) ? sbb_max : sb_bytes(fm);
    a.raw_xd_off = 128u * sbb_max;
    a.raw_stage = ((a.raw_xd_off + kRawXd) + 1023u) & ~1023u;
    a.hg = p.hg;
    a.hgd = p.hgd;
    a.hgsh = p.hgsh;
    a.hgsl = p.hgsl;
    if (p.keep_h) {
        a.h = f.h;
        a.hq = f.hq;
        a.hd = f.hd;
        a.hs = f.hs;
        a.hsum = f.hsum;
    }
    a.out = f.out;
    a.y = f.y;
    a.status = f.status;

    // activation-side maps over the slot-ordered operand of this phase
    CUtensorMap mx, md, msh, msl;
    const int K = a.K, slots = p.slots;
    const __half *xbase = p.phase == 0 ? p.xg : p.hg;
    const float *dbase = p.phase == 0 ? p.xgd : p.hgd;
    const float *shbase = p.phase == 0 ? p.xgsh : p.hgsh;
    const float *slbase = p.phase == 0 ? p.xgsl : p.hgsl;
    if (!encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, xbase, (uint64_t)K, (uint64_t)slots,
                   (uint64_t)K * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&md, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dbase, (uint64_t)(K / 32),
                   (uint64_t)slots, (uint64_t)(K / 32) * 4, 8, 32, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_2d(&msh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, shbase, (uint64_t)(K / 32),
                   (uint64_t)slots, (uint64_t)(K / 32) * 4, 8, 32, CU_TENSOR_MAP_SWIZZLE_32B) ||
        !encode_2d(&msl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, slbase, (uint64_t)(K / 32),
                   (uint64_t)slots, (uint64_t)(K / 32) * 4, 8, 32, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;

    const size_t smem = smem_bytes(a.raw_stage);
    const int grid = sm_count();
    if (grid <= 0) return cudaErrorInvalidDevice;
    cudaError_t err;
    if (p.phase == 0) {
        err = ensure_smem(k_gemm_tc<0>, smem);
        if (err != cudaSuccess) return err;
        k_gemm_tc<0><<<grid, kThreads, smem, st>>>(a, mx, md, msh, msl);
    } else {
        err = ensure_smem(k_gemm_tc<1>, smem);
        if (err != cudaSuccess) return err;
        k_gemm_tc<1><<<grid, kThreads, smem, st>>>(a, mx, md, msh, msl);
    }
    note_launches(1);
    err = cudaGetLastError();
    if (err != cudaSuccess && std::getenv("MOE_DEBUG")) {
        cudaFuncAttributes fa{};
        if (p.phase == 0) cudaFuncGetAttributes(&fa, k_gemm_tc<0>);
        else cudaFuncGetAttributes(&fa, k_gemm_tc<1>);
        std::fprintf(stderr,
                     "moe: k_gemm_tc<%d> launch failed: %s (regs %d, max threads %d, smem %zu)\n",
                     p.phase, cudaGetErrorString(err), fa.numRegs, fa.maxThreadsPerBlock, smem);
    }
    return err;
}

cudaError_t launch_act_gather(const int8_t *xq, const uint16_t *xd, const float *xsum,
                              const int32_t *perm, int T, int k, int H, int slots, __half *xg,
                              float *xgd, float *xgsh, float *xgsl, cudaStream_t st) {
    const int grid = (slots + 7) / 8;
    k_act_gather<<<grid, 256, 0, st>>>(xq, xd, xsum, perm, T, k, H, slots, xg, xgd, xgsh, xgsl);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_hg_tail_zero(__half *hg, float *hgd, float *hgsh, float *hgsl, int slots,
                                int F, int hpad, cudaStream_t st) {
    if (hpad == F) return cudaSuccess;
    k_hg_tail_zero<<<148, 256, 0, st>>>(hg, hgd, hgsh, hgsl, slots, F, hpad);
    note_launches(1);
    return cudaGetLastError();
}

size_t tc_smem_bytes(int fmt_mask) {
    uint32_t sbb_max = 0;
    for (int fm = 0; fm <= MOE_FMT_Q5_1; fm++)
        if (fmt_mask & (1 << fm)) sbb_max = sbb_max > sb_bytes(fm) ? sbb_max : sb_bytes(fm);
    const uint32_t raw_stage = ((128u * sbb_max + kRawXd) + 1023u) & ~1023u;
    return smem_bytes(raw_stage);
}

}  // namespace moe
