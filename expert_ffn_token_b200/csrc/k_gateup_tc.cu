// k_gateup_tc.cu -- a4 + a5 for large batches on the 5th-generation tensor cores (tcgen05):
// g = W_gate x^, u = W_up x^, h = silu(g) * u and Q8_1(h), for every (expert, token) pair.
//
// Prefill on the pages runs the routed experts as grouped matrix products over the tokens that
// share an expert ("Strata - the details", "Speed (measured)": "how many tokens share an expert",
// and the fused int8 tensor-core prompt experts of engine 0.1.36).  One persistent kernel, one
// CTA per SM, walks tiles of (expert job, up to 64 tokens, 128 values of f: the gate rows and the
// up rows of the same f).
//
// Arithmetic (exact products, fp32 sums).  h is re-quantized to Q8_1 before the down projection,
// and Q8_1 rounds every h to a multiple of its block's scale: an error of ~1e-4 in h moves many
// of those roundings and, through the down projection, the layer output by ~5e-3.  So g and u
// are computed as exactly as fp32 allows:
//   K-quant row, super-block sb: w = d * sc_j * q - dmin * m_j (sub-block j).  The operand A holds
//     the integers sc_j * q (<= 63 * 31, exact in fp16); the activation operand holds
//     x^ * 2^-e = xd_j * qx * 2^-e split into two fp16 values hi + lo that sum to it exactly.
//     Two MMAs per step (A * hi, A * lo) give P_sb = sum sc_j q x^ with exact products in the fp32
//     accumulator; the epilogue adds d_sb * P_sb once per super-block (one FFMA per element per
//     256 weights).  The min term sum_j RN32(dmin m_j) * xs_j (xs_j = xd_j * sum qx, the block
//     sum) is a contraction over the sub-blocks: kind::tf32 MMAs of hi/lo splits of both factors
//     (hi*hi + hi*lo + lo*hi, relative error ~2^-22) into its own accumulator.
//   Q8_0 / Q5_1 rows (w = d_b * q, w = d_b * q + m_b per 32 weights): A holds q, the epilogue
//     adds d_b * P_b once per 32-weight block, and Q5_1's offsets take the min term with -m_b.
// The epilogue multiplies by 2^e, forms h and quantizes it (a warp's 32 lanes are one 32-value
// block of f).
//
// Roles (512 threads, four warps per scheduler):
//   warp 0       TMA producer: per super-block the packed gate rows and up rows (128 each),
//                L2 prefetch two super-blocks ahead
//   warp 1       tensor-memory allocation and the MMA issuer
//   warps 2-5    unpack: thread r holds row r of gate and of up: the integer operands of every
//                64-wide stage, and per super-block the row scales and the min-term operands
//   warps 6-7    activation loader: gathers the tile's token rows (hi and lo planes, and the
//                block sums) with 16-byte cp.async, and the tile's column table
//   warps 8-15   epilogue: promotion, min term, SwiGLU, Q8_1(h)
// Every hand-off is an mbarrier; every wait is bounded and a timeout ends the kernel with
// MOE_ERR_TIMEOUT after the copies in flight have landed.
#include <cstdio>
#include <cstdlib>

#include "tc_pipe.cuh"

namespace moe {

namespace {

using namespace ptx;
using namespace tcp;

constexpr int kTN = 64;                          // tokens per tile
constexpr int kUnpackWarps = 4;
constexpr int kLoadWarp0 = 2 + kUnpackWarps;     // 6
constexpr int kLoadWarps = 2;
constexpr int kEpiWarp0 = kLoadWarp0 + kLoadWarps;   // 8
constexpr int kEpiWarps = 8;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;   // 512
constexpr uint32_t kAtomA = 16384;               // 128 rows x 64 fp16
constexpr uint32_t kAStage = 2 * kAtomA;         // gate, up
constexpr uint32_t kAtomB = kTN * 128;           // 64 token rows x 64 fp16
constexpr uint32_t kBStage = 2 * kAtomB;         // hi, lo
constexpr uint32_t kMinW = 128 * 32;             // 128 rows x 8 tf32 (32-byte swizzle)
constexpr uint32_t kMinX = kTN * 32;             // 64 token rows x 8 tf32
constexpr uint32_t kMStage = 4 * kMinW + 2 * kMinX;   // [g hi][g lo][u hi][u lo][x hi][x lo]
constexpr uint32_t kSStage = 2 * 8 * 128 * 2;    // row scales (fp16) [matrix][group][row]
constexpr int kMaxDA = 3, kMaxDB = 6, kMaxDR = 8;
constexpr uint32_t kTmemCols = 512;              // 2 x (gate | up) group buffers + 2 min buffers
constexpr size_t kSmemCap = 232448;

struct TileInfo {
    int tok[kTN];
    float w[kTN];
    float scale[kTN];
    int pad[kTN];
};

struct Smem {
    uint8_t *A, *B, *M, *raw;
    __half *scale;
    TileInfo *ti;
    uint64_t *raw_full, *raw_empty, *a_full, *a_empty, *b_full, *b_empty, *m_full, *m_empty,
        *s_full, *s_empty, *pg_full, *pg_empty, *tm_full, *tm_empty, *ti_full, *ti_empty, *done;
    uint32_t *tmem_slot;
    int *abort;
};

__host__ __device__ inline size_t smem_plan(int DA, int DB, int DR, uint32_t rawb) {
    return 1024 + (size_t)DA * kAStage + (size_t)DB * kBStage + 2 * kMStage + 2 * (size_t)kSStage +
           (size_t)DR * rawb + 2 * sizeof(TileInfo) +
           8 * (2 * kMaxDR + 2 * kMaxDA + 2 * kMaxDB + 21) + 16;
}

__device__ __forceinline__ Smem carve(uint8_t *base, const GemmArgs &a) {
    Smem s;
    uint8_t *p = base;
    s.A = p;
    p += (size_t)a.DA * kAStage;
    s.B = p;
    p += (size_t)a.DB * kBStage;
    s.M = p;
    p += 2 * kMStage;
    s.scale = reinterpret_cast<__half *>(p);
    p += 2 * (size_t)kSStage;
    s.raw = p;
    p += (size_t)a.DR * a.rawb;
    s.ti = reinterpret_cast<TileInfo *>(p);
    p += 2 * sizeof(TileInfo);
    uint64_t *b = reinterpret_cast<uint64_t *>(p);
    s.raw_full = b; b += kMaxDR;
    s.raw_empty = b; b += kMaxDR;
    s.a_full = b; b += kMaxDA;
    s.a_empty = b; b += kMaxDA;
    s.b_full = b; b += kMaxDB;
    s.b_empty = b; b += kMaxDB;
    s.m_full = b; b += 2;
    s.m_empty = b; b += 2;
    s.s_full = b; b += 2;
    s.s_empty = b; b += 2;
    s.pg_full = b; b += 2;
    s.pg_empty = b; b += 2;
    s.tm_full = b; b += 2;
    s.tm_empty = b; b += 2;
    s.ti_full = b; b += 2;
    s.ti_empty = b; b += 2;
    s.done = b; b += 1;
    s.tmem_slot = reinterpret_cast<uint32_t *>(b);
    s.abort = reinterpret_cast<int *>(b) + 1;
    return s;
}

__device__ __forceinline__ bool small_fmt(int fmt) {
    return fmt == MOE_FMT_Q8_0 || fmt == MOE_FMT_Q5_1;
}

// ---------------------------------------------------------------- warp 0: weight producer

__device__ void role_producer(const GemmArgs &a, const Smem &S, int nj, Ring &rr, int &issued) {
    Cursor cur;
    const int nsb = a.H / 256;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const CUtensorMap *m0 = a.wmaps + (size_t)t.e * 3 + 0, *m1 = a.wmaps + (size_t)t.e * 3 + 1;
        const int y = t.mt * 128;
        const uint32_t sbb = sb_bytes(t.fmt);
        const int xu = t.fmt == MOE_FMT_Q8_0 ? 136 : (int)sbb;   // Q8_0 maps count 16-bit units
        for (int sb = 0; sb < nsb; sb++) {
            if (sb + 2 < nsb) {
                tma_prefetch_2d(m0, (sb + 2) * xu, y);
                tma_prefetch_2d(m1, (sb + 2) * xu, y);
            }
            for (int hh = 0; hh < 2; hh++) {
                if (!wait1(a, S.abort, S.raw_empty + rr.s, rr.ph ^ 1u)) return;
                mbar_arrive_expect_tx(S.raw_full + rr.s, 128u * sbb);
                tma_load_2d(S.raw + (size_t)rr.s * a.rawb, hh ? m1 : m0, sb * xu, y,
                            S.raw_full + rr.s);
                issued++;
                rr.adv(1, a.DR);
            }
        }
    }
}

// ---------------------------------------------------------------- warps 2-5: unpack

// Integer operand values of one 64-wide stage of a row, in the operand order (0, 2, 1, 3) inside
// every 4.  K-quants: sc_j * q for sub-blocks 2st (low nibbles of qs[32st .. 32st+32)) and 2st+1
// (high nibbles), fma(1024 + q, sc, -1024 sc) being exact.  Q8_0: q of blocks 2st, 2st+1.
// Q5_1: q (0..31) of blocks 2st, 2st+1.
template <int FMT>
__device__ __forceinline__ void int_stage(const uint8_t *rowp, int st, uint32_t scp,
                                          const uint32_t (&qh)[8], uint32_t (&v)[32]) {
    constexpr uint32_t kM = 0x000F000Fu, kE = 0x64006400u;
    if (FMT == MOE_FMT_Q4_K || FMT == MOE_FMT_Q5_K) {
        const uint4 *qp = reinterpret_cast<const uint4 *>(rowp + (FMT == MOE_FMT_Q5_K ? 48 : 16) +
                                                          32 * st);
        const uint4 qa = qp[0], qb = qp[1];
        const uint32_t qw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
        const __half2 sp = u2h(scp);
        const __half2 s0 = __low2half2(sp), s1 = __high2half2(sp);
        const __half2 k1024 = __float2half2_rn(-1024.0f);
        const __half2 n0 = __hmul2(s0, k1024), n1 = __hmul2(s1, k1024);
#pragma unroll
        for (int wi = 0; wi < 8; wi++) {
            const uint32_t x = qw[wi];
            uint32_t la = lop3_and_or(x, kM, kE), lb = lop3_and_or(x >> 8, kM, kE);
            uint32_t ha = lop3_and_or(x >> 4, kM, kE), hb = lop3_and_or(x >> 12, kM, kE);
            if (FMT == MOE_FMT_Q5_K) {   // fifth bits: bit 2st (low nibbles), 2st+1 (high)
                const uint32_t t = qh[wi] >> (2 * st);
                la |= (t << 4) & 0x00100010u;
                lb |= (t >> 4) & 0x00100010u;
                ha |= (t << 3) & 0x00100010u;
                hb |= (t >> 5) & 0x00100010u;
            }
            v[2 * wi] = h2u(__hfma2(u2h(la), s0, n0));
            v[2 * wi + 1] = h2u(__hfma2(u2h(lb), s0, n0));
            v[16 + 2 * wi] = h2u(__hfma2(u2h(ha), s1, n1));
            v[16 + 2 * wi + 1] = h2u(__hfma2(u2h(hb), s1, n1));
        }
    } else if (FMT == MOE_FMT_Q8_0) {
        const __half2 k1152 = __float2half2_rn(1152.0f);
#pragma unroll
        for (int bb = 0; bb < 2; bb++) {
            const uint8_t *blk = rowp + 34 * (2 * st + bb);
            uint32_t q[8];
            if (bb == 0) {   // quants start 2 bytes past a word boundary
                const uint32_t *wp = reinterpret_cast<const uint32_t *>(blk);
                uint32_t wv[9];
#pragma unroll
                for (int i = 0; i < 9; i++) wv[i] = wp[i];
#pragma unroll
                for (int i = 0; i < 8; i++) q[i] = __funnelshift_r(wv[i], wv[i + 1], 16);
            } else {
                const uint32_t *wp = reinterpret_cast<const uint32_t *>(blk + 2);
#pragma unroll
                for (int i = 0; i < 8; i++) q[i] = wp[i];
            }
#pragma unroll
            for (int i = 0; i < 8; i++) {
                // byte b -> fp16 (1024 + (b ^ 0x80)) - 1152 = b, exactly
                const uint32_t x = q[i] ^ 0x80808080u;
                v[16 * bb + 2 * i] = h2u(__hsub2(u2h(prmt(x, 0x64646464u, 0x4240u)), k1152));
                v[16 * bb + 2 * i + 1] = h2u(__hsub2(u2h(prmt(x, 0x64646464u, 0x4341u)), k1152));
            }
        }
    } else {   // Q5_1
        const __half2 k1024 = __float2half2_rn(1024.0f);
#pragma unroll
        for (int bb = 0; bb < 2; bb++) {
            const uint2 *bp = reinterpret_cast<const uint2 *>(rowp + 24 * (2 * st + bb));
            const uint2 h = bp[0], qa = bp[1], qb = bp[2];
            const uint32_t qw[4] = {qa.x, qa.y, qb.x, qb.y};
#pragma unroll
            for (int wi = 0; wi < 8; wi++) {
                // elements 4wi..4wi+3: n < 16 low nibbles of qs[n], n >= 16 high of qs[n-16]
                const uint32_t x = wi < 4 ? qw[wi] : qw[wi - 4] >> 4;
                const uint32_t t = h.y >> (4 * wi);
                const uint32_t pa = lop3_and_or(x, kM, kE) | (((t & 5u) * 0x40010u) & 0x00100010u);
                const uint32_t pb =
                    lop3_and_or(x >> 8, kM, kE) | (((t & 10u) * 0x20008u) & 0x00100010u);
                v[16 * bb + 2 * wi] = h2u(__hsub2(u2h(pa), k1024));
                v[16 * bb + 2 * wi + 1] = h2u(__hsub2(u2h(pb), k1024));
            }
        }
    }
}

// Per super-block constants of one row: the promotion scale of each group (d, or d_b per
// 32-weight block), the min-term weights wm_j (RN32(dmin m_j), or -m_b for Q5_1) and the
// integer scales sc_j as fp16 pairs (K-quants).
template <int FMT>
__device__ __forceinline__ void row_consts(const uint8_t *rowp, float (&dsc)[8], float (&wm)[8],
                                           uint32_t (&scp)[4], uint32_t (&qh)[8]) {
    if (FMT == MOE_FMT_Q4_K || FMT == MOE_FMT_Q5_K) {
        const uint4 hdr = *reinterpret_cast<const uint4 *>(rowp);
        const float d = half_bits_to_float(hdr.x), dmin = half_bits_to_float(hdr.x >> 16);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            int sc0, mn0, sc1, mn1;
            kq_scale_min(hdr.y, hdr.z, hdr.w, j, sc0, mn0);
            kq_scale_min(hdr.y, hdr.z, hdr.w, j + 1, sc1, mn1);
            scp[j / 2] = h2u(__floats2half2_rn((float)sc0, (float)sc1));
            wm[j] = __fmul_rn(dmin, (float)mn0);
            wm[j + 1] = __fmul_rn(dmin, (float)mn1);
        }
#pragma unroll
        for (int j = 0; j < 8; j++) dsc[j] = d;
        if (FMT == MOE_FMT_Q5_K) {
            const uint4 *hp = reinterpret_cast<const uint4 *>(rowp + 16);
            const uint4 ha = hp[0], hb = hp[1];
            qh[0] = ha.x; qh[1] = ha.y; qh[2] = ha.z; qh[3] = ha.w;
            qh[4] = hb.x; qh[5] = hb.y; qh[6] = hb.z; qh[7] = hb.w;
        }
    } else {
#pragma unroll
        for (int b = 0; b < 8; b++) {
            const uint8_t *blk = rowp + (FMT == MOE_FMT_Q8_0 ? 34 : 24) * b;
            dsc[b] = half_bits_to_float(*reinterpret_cast<const uint16_t *>(blk));
            wm[b] = FMT == MOE_FMT_Q5_1
                        ? -half_bits_to_float(*reinterpret_cast<const uint16_t *>(blk + 2))
                        : 0.0f;
        }
    }
}

// Row r of a min-term weight region (8 tf32, 32-byte swizzle: chunk c at c ^ ((r >> 2) & 1)).
__device__ __forceinline__ void store_min_row(uint8_t *region, int r, const float (&v)[8]) {
    float4 *p = reinterpret_cast<float4 *>(region + r * 32);
    const int sw = (r >> 2) & 1;
    p[0 ^ sw] = make_float4(v[0], v[1], v[2], v[3]);
    p[1 ^ sw] = make_float4(v[4], v[5], v[6], v[7]);
}

template <int FMT>
__device__ __forceinline__ bool unpack_sb(const GemmArgs &a, const Smem &S, Ring &ra, Ring &rs,
                                          Ring &rm, const uint8_t *rowg, const uint8_t *rowu,
                                          int r) {
    const int lane = threadIdx.x & 31;
    float dg[8], du[8], wg[8], wu[8];
    uint32_t scg[4] = {0, 0, 0, 0}, scu[4] = {0, 0, 0, 0};
    uint32_t qhg[8] = {0, 0, 0, 0, 0, 0, 0, 0}, qhu[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    row_consts<FMT>(rowg, dg, wg, scg, qhg);
    row_consts<FMT>(rowu, du, wu, scu, qhu);
    // promotion scales of this super-block's groups
    if (!waitw(a, S.abort, S.s_empty + rs.s, rs.ph ^ 1u)) return false;
    __half *sc = S.scale + (size_t)rs.s * (kSStage / 2);
    const int ng = small_fmt(FMT) ? 8 : 1;
#pragma unroll
    for (int g = 0; g < 8; g++) {
        if (g < ng) {   // the scales are fp16 values of the blocks: exact as __half
            sc[(0 * 8 + g) * 128 + r] = __float2half_rn(dg[g]);
            sc[(1 * 8 + g) * 128 + r] = __float2half_rn(du[g]);
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(S.s_full + rs.s);
    rs.adv(1, 2);
    // min-term weights, split into tf32 hi + lo
    if (has_min(FMT)) {
        if (!waitw(a, S.abort, S.m_empty + rm.s, rm.ph ^ 1u)) return false;
        float hi[8], lo[8];
#pragma unroll
        for (int j = 0; j < 8; j++) {
            hi[j] = tf32_round(wg[j]);
            lo[j] = tf32_round(wg[j] - hi[j]);
        }
        uint8_t *ms = S.M + (size_t)rm.s * kMStage;
        store_min_row(ms + 0 * kMinW, r, hi);
        store_min_row(ms + 1 * kMinW, r, lo);
#pragma unroll
        for (int j = 0; j < 8; j++) {
            hi[j] = tf32_round(wu[j]);
            lo[j] = tf32_round(wu[j] - hi[j]);
        }
        store_min_row(ms + 2 * kMinW, r, hi);
        store_min_row(ms + 3 * kMinW, r, lo);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(S.m_full + rm.s);
        rm.adv(1, 2);
    }
    // the four 64-wide stages
#pragma unroll 1
    for (int st = 0; st < 4; st++) {
        if (!waitw(a, S.abort, S.a_empty + ra.s, ra.ph ^ 1u)) return false;
        uint8_t *as = S.A + (size_t)ra.s * kAStage;
        uint32_t v[32];
        const uint32_t sg = st == 0 ? scg[0] : st == 1 ? scg[1] : st == 2 ? scg[2] : scg[3];
        const uint32_t su = st == 0 ? scu[0] : st == 1 ? scu[1] : st == 2 ? scu[2] : scu[3];
        int_stage<FMT>(rowg, st, sg, qhg, v);
        store_row(as, r, v);
        int_stage<FMT>(rowu, st, su, qhu, v);
        store_row(as + kAtomA, r, v);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(S.a_full + ra.s);
        ra.adv(1, a.DA);
    }
    return true;
}

__device__ void role_unpack(const GemmArgs &a, const Smem &S, int nj) {
    const int r = threadIdx.x - 64;          // 0..127: row r of gate and of up
    const int lane = threadIdx.x & 31;
    Cursor cur;
    Ring rr, ra, rs, rm;
    const int nsb = a.H / 256;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const uint32_t sbb = sb_bytes(t.fmt);
        for (int sb = 0; sb < nsb; sb++) {
            Ring ru = rr;
            ru.adv(1, a.DR);                 // the up rows' packed stage follows the gate rows'
            if (!waitw(a, S.abort, S.raw_full + rr.s, rr.ph)) return;
            if (!waitw(a, S.abort, S.raw_full + ru.s, ru.ph)) return;
            const uint8_t *rowg = S.raw + (size_t)rr.s * a.rawb + (size_t)r * sbb;
            const uint8_t *rowu = S.raw + (size_t)ru.s * a.rawb + (size_t)r * sbb;
            bool ok;
            if (t.fmt == MOE_FMT_Q4_K) ok = unpack_sb<MOE_FMT_Q4_K>(a, S, ra, rs, rm, rowg, rowu, r);
            else if (t.fmt == MOE_FMT_Q5_K) ok = unpack_sb<MOE_FMT_Q5_K>(a, S, ra, rs, rm, rowg, rowu, r);
            else if (t.fmt == MOE_FMT_Q8_0) ok = unpack_sb<MOE_FMT_Q8_0>(a, S, ra, rs, rm, rowg, rowu, r);
            else ok = unpack_sb<MOE_FMT_Q5_1>(a, S, ra, rs, rm, rowg, rowu, r);
            if (!ok) return;
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(S.raw_empty + rr.s);
                mbar_arrive(S.raw_empty + ru.s);
            }
            rr.adv(2, a.DR);
        }
    }
}

// ---------------------------------------------------------------- warp 1: MMA issuer

__device__ void role_mma(const GemmArgs &a, const Smem &S, int nj, uint32_t tbase) {
    Cursor cur;
    Ring ra, rb, rm, rg, rt;
    const uint32_t a_base = smem_u32(S.A), b_base = smem_u32(S.B), m_base = smem_u32(S.M);
    const int nsb = a.H / 256;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const uint32_t idf = instr_desc(0, 128, t.n_mma);
        const uint32_t idt = instr_desc(2, 128, t.n_mma);
        const bool small = small_fmt(t.fmt), mn = has_min(t.fmt);
        if (!wait1(a, S.abort, S.tm_empty + rt.s, rt.ph ^ 1u)) return;
        tc_fence_after();
        const uint32_t dmin = tbase + 256 + (uint32_t)rt.s * 128;   // gate min, up min at +64
        for (int sb = 0; sb < nsb; sb++) {
            for (int st = 0; st < 4; st++) {
                if (!wait1(a, S.abort, S.a_full + ra.s, ra.ph)) return;
                if (!wait1(a, S.abort, S.b_full + rb.s, rb.ph)) return;
                tc_fence_after();
                const uint64_t dAg = smem_desc(a_base + (uint32_t)ra.s * kAStage, 1024, 2);
                const uint64_t dAu = smem_desc(a_base + (uint32_t)ra.s * kAStage + kAtomA, 1024, 2);
                const uint64_t dBh = smem_desc(b_base + (uint32_t)rb.s * kBStage, 1024, 2);
                const uint64_t dBl = smem_desc(b_base + (uint32_t)rb.s * kBStage + kAtomB, 1024, 2);
#pragma unroll
                for (int kk = 0; kk < 4; kk++) {
                    // a group starts at K-step 0 of each super-block (K-quants) or of each
                    // 32-weight block (kk = 0, 2; Q8_0 and Q5_1)
                    const bool first = small ? (kk & 1) == 0 : (st == 0 && kk == 0);
                    if (first) {
                        if (!wait1(a, S.abort, S.pg_empty + rg.s, rg.ph ^ 1u)) return;
                        tc_fence_after();
                    }
                    const uint32_t dg = tbase + (uint32_t)rg.s * 128, du = dg + 64;
                    const uint32_t acc = first ? 0u : 1u;
                    umma_f16(dg, dAg + 2 * kk, dBh + 2 * kk, idf, acc);
                    umma_f16(dg, dAg + 2 * kk, dBl + 2 * kk, idf, 1u);
                    umma_f16(du, dAu + 2 * kk, dBh + 2 * kk, idf, acc);
                    umma_f16(du, dAu + 2 * kk, dBl + 2 * kk, idf, 1u);
                    const bool last = small ? (kk & 1) == 1 : (st == 3 && kk == 3);
                    if (last) {
                        umma_commit(S.pg_full + rg.s);
                        rg.adv(1, 2);
                    }
                }
                umma_commit(S.a_empty + ra.s);
                umma_commit(S.b_empty + rb.s);
                ra.adv(1, a.DA);
                rb.adv(1, a.DB);
            }
            if (mn) {   // the min term of this super-block, after its main products (its operands
                        // came with the super-block's first stage, so they have landed by now)
                if (!wait1(a, S.abort, S.m_full + rm.s, rm.ph)) return;
                tc_fence_after();
                const uint32_t mb = m_base + (uint32_t)rm.s * kMStage;
                const uint64_t wgh = smem_desc(mb + 0 * kMinW, 256, 6);
                const uint64_t wgl = smem_desc(mb + 1 * kMinW, 256, 6);
                const uint64_t wuh = smem_desc(mb + 2 * kMinW, 256, 6);
                const uint64_t wul = smem_desc(mb + 3 * kMinW, 256, 6);
                const uint64_t xh = smem_desc(mb + 4 * kMinW, 256, 6);
                const uint64_t xl = smem_desc(mb + 4 * kMinW + kMinX, 256, 6);
                const uint32_t acc0 = sb > 0 ? 1u : 0u;
                umma_tf32(dmin, wgh, xh, idt, acc0);
                umma_tf32(dmin, wgh, xl, idt, 1u);
                umma_tf32(dmin, wgl, xh, idt, 1u);
                umma_tf32(dmin + 64, wuh, xh, idt, acc0);
                umma_tf32(dmin + 64, wuh, xl, idt, 1u);
                umma_tf32(dmin + 64, wul, xh, idt, 1u);
                umma_commit(S.m_empty + rm.s);
                rm.adv(1, 2);
            }
        }
        umma_commit(S.tm_full + rt.s);
        rt.adv(1, 2);
    }
}

// ---------------------------------------------------------------- warps 6-7: activation loader

__device__ void role_loader(const GemmArgs &a, const Smem &S, int nj) {
    const int lt = threadIdx.x - kLoadWarp0 * 32;   // 0..63
    const int lane = lt & 31;
    const int c = lt & 7;                        // 16-byte chunk of a 128-byte row
    const int rg = lt >> 3;                      // rows rg + 8 j, j = 0..7
    Cursor cur;
    Ring rb, rt, rm;
    // stages issued but not yet signalled are consecutive: the oldest one's B and M positions
    Ring ob, om;
    int og = 0, npend = 0;
    bool ok = true;
    const int nsb = a.H / 256;
    const int H32 = a.H / 32;
    for (int i = blockIdx.x; ok; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        if (!(ok = waitw(a, S.abort, S.ti_empty + rt.s, rt.ph ^ 1u))) break;
        TileInfo &ti = S.ti[rt.s];
        int my_tok = -1;                         // token of column lt (for the block sums)
        if (lt < t.n_valid) {
            const int slot = t.slot_base + lt;
            float wt;
            if (t.shared) {
                my_tok = slot - a.T * a.k;
                wt = 1.0f;
            } else {
                const int p = a.perm[slot];
                my_tok = p / a.k;
                wt = a.w[p];
            }
            ti.tok[lt] = my_tok;
            ti.w[lt] = wt;
            ti.scale[lt] = a.act_scale[my_tok];
        }
        int src[8];                              // this thread's gather rows
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int n = rg + 8 * j;
            src[j] = -1;
            if (n < t.n_valid) {
                const int slot = t.slot_base + n;
                src[j] = t.shared ? slot - a.T * a.k : a.perm[slot] / a.k;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(S.ti_full + rt.s);
        rt.adv(1, 2);
        const bool mn = has_min(t.fmt);
        ob = rb;
        om = rm;
        og = 0;
        // signal the oldest issued stage (its copies have landed): B, and the block sums it
        // carried at a super-block's first stage
        auto signal_oldest = [&]() {
            if (lane == 0) {
                mbar_arrive(S.b_full + ob.s);
                if (mn && (og & 3) == 0) mbar_arrive(S.m_full + om.s);
            }
            if (mn && (og & 3) == 0) om.adv(1, 2);
            ob.adv(1, a.DB);
            og++;
            npend--;
        };
        for (int sb = 0; sb < nsb && ok; sb++) {
            for (int st = 0; st < 4; st++) {
                if (st == 0 && mn) {   // the block sums of this super-block (min-term operand)
                    if (!(ok = waitw(a, S.abort, S.m_empty + rm.s, rm.ph ^ 1u))) break;
                    if (my_tok >= 0) {
                        const int sw = (lt >> 2) & 1;
                        const float *hs = a.xs_hi + (size_t)my_tok * H32 + 8 * sb;
                        const float *ls = a.xs_lo + (size_t)my_tok * H32 + 8 * sb;
                        uint8_t *xh = S.M + (size_t)rm.s * kMStage + 4 * kMinW + lt * 32;
                        cp_async16(xh + ((0 ^ sw) << 4), hs);
                        cp_async16(xh + ((1 ^ sw) << 4), hs + 4);
                        cp_async16(xh + kMinX + ((0 ^ sw) << 4), ls);
                        cp_async16(xh + kMinX + ((1 ^ sw) << 4), ls + 4);
                    }
                    rm.adv(1, 2);
                }
                if (!(ok = waitw(a, S.abort, S.b_empty + rb.s, rb.ph ^ 1u))) break;
                uint8_t *bs = S.B + (size_t)rb.s * kBStage;
                const int g = 4 * sb + st;
                const __half *colh = a.act + 64 * g + 8 * c;
                const __half *coll = a.act_lo + 64 * g + 8 * c;
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const int n = rg + 8 * j;
                    if (src[j] >= 0) {
                        const uint32_t off = (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4);
                        cp_async16(bs + off, colh + (size_t)src[j] * a.act_pitch);
                        cp_async16(bs + kAtomB + off, coll + (size_t)src[j] * a.act_pitch);
                    }
                }
                cp_async_commit();
                npend++;
                rb.adv(1, a.DB);
                if (npend > a.lag) {
                    if (a.lag >= 4) cp_async_wait<4>();
                    else if (a.lag == 3) cp_async_wait<3>();
                    else if (a.lag == 2) cp_async_wait<2>();
                    else cp_async_wait<1>();
                    fence_proxy_async_smem();
                    __syncwarp();
                    signal_oldest();
                }
            }
        }
        // the tile's last stages: land them now rather than after the next tile's set-up
        cp_async_wait<0>();
        fence_proxy_async_smem();
        __syncwarp();
        while (npend > 0) signal_oldest();
    }
    cp_async_wait<0>();
}

// ---------------------------------------------------------------- warps 8-15: epilogue

__device__ void role_epilogue(const GemmArgs &a, const Smem &S, int nj, uint32_t tbase) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;                  // tensor-memory lane quarter: rows 32q + lane
    const int ch = (warp - kEpiWarp0) >> 2;  // columns (tokens) 32ch .. 32ch + 31
    const int r = 32 * q + lane;
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    Cursor cur;
    Ring rs, rg, rt;
    const int nsb = a.H / 256;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const bool small = small_fmt(t.fmt), mn = has_min(t.fmt);
        const int ng = small ? 8 : 1;
        float tg[32], tu[32];
#pragma unroll
        for (int j = 0; j < 32; j++) tg[j] = tu[j] = 0.0f;
        for (int sb = 0; sb < nsb; sb++) {
            if (!waitw(a, S.abort, S.s_full + rs.s, rs.ph)) return;
            const __half *sc = S.scale + (size_t)rs.s * (kSStage / 2);
            for (int g = 0; g < ng; g++) {
                const float dg = __half2float(sc[(0 * 8 + g) * 128 + r]);
                const float du = __half2float(sc[(1 * 8 + g) * 128 + r]);
                if (!waitw(a, S.abort, S.pg_full + rg.s, rg.ph)) return;
                tc_fence_after();
                const uint32_t col = tbase + lane_addr + (uint32_t)rg.s * 128 + 32 * ch;
#pragma unroll
                for (int hf = 0; hf < 2; hf++) {   // 16 columns at a time: fewer live registers
                    uint32_t P[16];
                    tmem_ld16(col + 16 * hf, P);
                    tmem_ld_wait(P);
#pragma unroll
                    for (int j = 0; j < 16; j++)
                        tg[16 * hf + j] = fmaf(dg, __uint_as_float(P[j]), tg[16 * hf + j]);
                    tmem_ld16(col + 64 + 16 * hf, P);
                    tmem_ld_wait(P);
#pragma unroll
                    for (int j = 0; j < 16; j++)
                        tu[16 * hf + j] = fmaf(du, __uint_as_float(P[j]), tu[16 * hf + j]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(S.pg_empty + rg.s);
                rg.adv(1, 2);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(S.s_empty + rs.s);
            rs.adv(1, 2);
        }
        if (!waitw(a, S.abort, S.tm_full + rt.s, rt.ph)) return;
        tc_fence_after();
        if (mn) {
            const uint32_t col = tbase + lane_addr + 256 + (uint32_t)rt.s * 128 + 32 * ch;
#pragma unroll
            for (int hf = 0; hf < 2; hf++) {
                uint32_t P[16];
                tmem_ld16(col + 16 * hf, P);
                tmem_ld_wait(P);
#pragma unroll
                for (int j = 0; j < 16; j++) tg[16 * hf + j] -= __uint_as_float(P[j]);
                tmem_ld16(col + 64 + 16 * hf, P);
                tmem_ld_wait(P);
#pragma unroll
                for (int j = 0; j < 16; j++) tu[16 * hf + j] -= __uint_as_float(P[j]);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(S.tm_empty + rt.s);
        if (!waitw(a, S.abort, S.ti_full + rt.s, rt.ph)) return;
        const TileInfo &ti = S.ti[rt.s];
        const int f = 128 * t.mt + r;
        const int nc = min(32, t.n_valid - 32 * ch);
        if (128 * t.mt + 32 * q < a.F) {   // the warp's 32 rows are one block of f, in range
#pragma unroll
            for (int j = 0; j < 32; j++) {
                if (j < nc) {
                    const int n = 32 * ch + j;
                    const float s = ti.scale[n];
                    const float h = silu_mul(tg[j] * s, tu[j] * s);
                    quantize_h_lane(a, h, t.slot_base + n, f);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(S.ti_empty + rt.s);
        rt.adv(1, 2);
    }
}

// ---------------------------------------------------------------- the kernel

__global__ void __launch_bounds__(kThreads, 1) k_gateup_tc(const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const Smem S = carve(base, a);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.DR; i++) {
            mbar_init(S.raw_full + i, 1);
            mbar_init(S.raw_empty + i, kUnpackWarps);
        }
        for (int i = 0; i < a.DA; i++) {
            mbar_init(S.a_full + i, kUnpackWarps);
            mbar_init(S.a_empty + i, 1);
        }
        for (int i = 0; i < a.DB; i++) {
            mbar_init(S.b_full + i, kLoadWarps);
            mbar_init(S.b_empty + i, 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(S.m_full + i, kUnpackWarps + kLoadWarps);
            mbar_init(S.m_empty + i, 1);
            mbar_init(S.s_full + i, kUnpackWarps);
            mbar_init(S.s_empty + i, kEpiWarps);
            mbar_init(S.pg_full + i, 1);
            mbar_init(S.pg_empty + i, kEpiWarps);
            mbar_init(S.tm_full + i, 1);
            mbar_init(S.tm_empty + i, kEpiWarps);
            mbar_init(S.ti_full + i, kLoadWarps);
            mbar_init(S.ti_empty + i, kEpiWarps);
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
        if (lane == 0) {
            Ring rr;
            int issued = 0;
            role_producer(a, S, nj, rr, issued);
            if (*(volatile int *)S.abort) {
                // the loads already issued land before the CTA leaves (each wait bounded): walk
                // back over the last positions filled, one ring's worth at most
                const int n = issued < a.DR ? issued : a.DR;
                for (int k = 0; k < n; k++) {
                    if (--rr.s < 0) {
                        rr.s = a.DR - 1;
                        rr.ph ^= 1u;
                    }
                    mbar_wait_bounded(S.raw_full + rr.s, rr.ph, 20000000ull);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            role_mma(a, S, nj, tbase);
            umma_commit(S.done);
            mbar_wait_bounded(S.done, 0, 20000000ull);
        }
        __syncwarp();
    } else if (warp < kLoadWarp0) {
        role_unpack(a, S, nj);
        __syncwarp();
    } else if (warp < kEpiWarp0) {
        role_loader(a, S, nj);
        __syncwarp();
    } else {
        role_epilogue(a, S, nj, tbase);
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

uint32_t raw_bytes(int fmt_mask) {
    uint32_t sbb_max = 0;
    for (int fm = 0; fm <= MOE_FMT_Q5_1; fm++)
        if (fmt_mask & (1 << fm)) sbb_max = sbb_max > sb_bytes(fm) ? sbb_max : sb_bytes(fm);
    return ((128u * sbb_max) + 1023u) & ~1023u;
}

// Ring depths that fit the shared memory: two integer-operand stages, the deepest activation
// ring (five down to two stages: the gathers come from L2 and want several stages in flight)
// that leaves room for three packed half-stages (one and a half super-blocks), else the deepest
// one with one super-block of packed rows (the 272-byte Q8_0 super-blocks need that).
bool ring_plan(int fmt_mask, int &DA, int &DB, int &DR) {
    const uint32_t rawb = raw_bytes(fmt_mask);
    DA = 2;
    for (int need = 3; need >= 2; need--) {
        for (DB = 5; DB >= 2; DB--) {
            const size_t fixed = smem_plan(DA, DB, 0, rawb);
            if (fixed >= kSmemCap) continue;
            DR = (int)((kSmemCap - fixed) / rawb);
            if (DR > kMaxDR) DR = kMaxDR;
            if (DR >= need) return true;
        }
    }
    return false;
}

}  // namespace

size_t tc_gateup_smem_bytes(int fmt_mask) {
    int DA, DB, DR;
    if (!ring_plan(fmt_mask, DA, DB, DR)) return (size_t)-1;
    return smem_plan(DA, DB, DR, raw_bytes(fmt_mask));
}

cudaError_t launch_gateup_tc(const TcPhaseArgs &p, int grid, cudaStream_t st) {
    const FfnArgs &f = p.ffn;
    GemmArgs a{};
    a.wmaps = reinterpret_cast<const CUtensorMap *>(p.wmaps);
    a.experts = f.experts;
    a.jobs = f.jobs;
    a.njobs = f.njobs;
    a.perm = f.perm;
    a.w = f.w;
    a.act = p.xh;
    a.act_lo = p.xl;
    a.xs_hi = p.xsh;
    a.xs_lo = p.xsl;
    a.act_scale = p.xscale;
    a.act_pitch = f.H;
    a.T = f.T;
    a.k = f.k;
    a.H = f.H;
    a.F = f.F;
    a.hpad = f.hpad;
    a.nst = f.H / 64;
    a.mt_count = (f.F + 127) / 128;
    a.tn = kTN;
    if (!ring_plan(f.fmt_mask, a.DA, a.DB, a.DR)) return cudaErrorInvalidValue;
    a.lag = a.DB - 1;
    a.rawb = raw_bytes(f.fmt_mask);
    a.hq = f.hq;
    a.hd = f.hd;
    a.hs = f.hs;
    a.hsum = f.hsum;
    a.h = p.keep_h ? f.h : nullptr;
    a.status = f.status;
    a.wait_ns = p.wait_ns;
    const size_t smem = smem_plan(a.DA, a.DB, a.DR, a.rawb);
    if (grid <= 0) return cudaErrorInvalidDevice;
    cudaError_t err = ensure_smem(k_gateup_tc, smem);
    if (err != cudaSuccess) return err;
    if (std::getenv("MOE_DEBUG"))
        std::fprintf(stderr, "moe: k_gateup_tc grid %d smem %zu rings %d/%d/%d rawb %u\n", grid,
                     smem, a.DA, a.DB, a.DR, a.rawb);
    k_gateup_tc<<<grid, kThreads, smem, st>>>(a);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
