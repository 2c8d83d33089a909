// k_gateup_i8.cu -- a4 + a5 for large batches with 8-bit integer tensor-core products
// (tcgen05.mma kind::i8): g = W_gate x^, u = W_up x^, h = silu(g) * u and Q8_1(h), for every
// (expert, token) pair.  The same tiles, outputs and roles as k_gateup_tc.cu; only the arithmetic
// differs.
//
// The pages run the prompt's experts as fused int8 tensor-core kernels ("Strata - the details",
// "Speed (measured)", engine 0.1.36): the packed weights' integer quants against the int8 quants
// of Q8_1(x).  Here, for every 32-weight block b of a row and every token t:
//   I_tb = sum_i q_i * qx_ti          (exact, one K = 32 MMA into its own s32 accumulator)
// and the epilogue promotes each block once:
//   acc_t += I_tb * (s_b * xd_tb) - wm_b * xs_tb
// with s_b the block's weight scale (d * sc_j for K-quants, d_b for Q8_0 and Q5_1), wm_b its min
// term (RN32(dmin * m_j); -m_b for Q5_1; 0 for Q8_0), xd_tb the activation block scale and xs_tb
// = xd_tb * sum(qx), the block sum.  The products wm_b * xs_tb and the integer I_tb are exact in
// fp32; s_b * xd_tb rounds once; every term is added with one rounding.
//
// Cost model.  One MMA per 32 weights per matrix (kind::f16 with exact operands needs four per
// 16), so the tensor pipe is nowhere near busy; the epilogue's per-block promotion is the work:
// per element and block a conversion and three fp32 operations (the scale product, the product
// and the min term), the fp32 ones issued as packed f32x2 pairs.
//
// Roles (640 threads, 96 registers each):
//   warp 0       TMA producer: per super-block the packed gate rows and up rows (128 each), L2
//                prefetch two super-blocks ahead
//   warp 1       tensor-memory allocation and the MMA issuer: per 32-weight block two MMAs (gate,
//                up) into one of four rotating accumulator slots of 64 + 64 columns
//   warp 2       loader: the tile's token rows of Q8_1(x) gathered with 16-byte cp.async, per
//                stage the columns' block scales and block sums (loaded a stage ahead), and the
//                block constants (s_b, -wm_b) of rows lane + 32 i read from the packed rows
//   warp 3       unpack: lane u holds rows u + 32 i (i = 0..3) of gate and of up: their int8
//                operands of every 128-wide stage
//   warps 4-19   epilogue: four warps per tensor-memory lane quarter, 16 tokens each: promotion,
//                SwiGLU, Q8_1(h)
// Every hand-off is an mbarrier; every wait is bounded and a timeout ends the kernel with
// MOE_ERR_TIMEOUT after the copies in flight have landed.
#include <cstdio>
#include <cstdlib>

#include "tc_pipe.cuh"

namespace moe {

namespace {

using namespace ptx;
using namespace tcp;

constexpr int kTN = 64;                              // tokens per tile
constexpr int kLoadWarp = 2;
constexpr int kUnpackWarp = 3;
constexpr int kEpiWarp0 = 4;
constexpr int kEpiCols = 16;                         // tokens per epilogue warp
constexpr int kEpiWarps = 4 * kTN / kEpiCols;        // four lane quarters x the tile's tokens
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;   // 640: five warps per scheduler
constexpr uint32_t kAtomA = 16384;                   // 128 rows x 128 int8
constexpr uint32_t kAStage = 2 * kAtomA;             // gate, up
constexpr uint32_t kBStage = kTN * 128;              // 64 token rows x 128 int8
constexpr uint32_t kKStage = 4 * 128 * 16;           // [block][row] {s_g, s_u, -wm_g, -wm_u}
constexpr uint32_t kCStage = 2 * 4 * kTN * 4;        // [block][token] xd, then [block][token] xs
constexpr int kSlots = 4;                            // accumulator slots of 128 columns
constexpr int kMaxDR = 8, kMaxDA = 2, kMaxDB = 4, kMaxDK = 4, kMaxDC = 6;
constexpr uint32_t kTmemCols = 512;
constexpr size_t kSmemCap = 232448;

struct Smem {
    uint8_t *A, *B, *raw;
    float4 *kc;
    float *cc;
    uint64_t *raw_full, *raw_empty, *a_full, *a_empty, *b_full, *b_empty, *k_full, *k_empty,
        *c_full, *c_empty, *s_full, *s_empty, *done;
    uint32_t *tmem_slot;
    int *abort;
};

__host__ __device__ inline size_t smem_plan(int DB, int DK, int DC, int DR, uint32_t rawb) {
    return 1024 + (size_t)kMaxDA * kAStage + (size_t)DB * kBStage + (size_t)DK * kKStage +
           (size_t)DC * kCStage + (size_t)DR * rawb +
           8 * (2 * kMaxDR + 2 * kMaxDA + 2 * kMaxDB + 2 * kMaxDK + 2 * kMaxDC + 2 * kSlots + 1) +
           16;
}

__device__ __forceinline__ Smem carve(uint8_t *base, const GemmArgs &a) {
    Smem s;
    uint8_t *p = base;
    s.A = p;
    p += (size_t)kMaxDA * kAStage;
    s.B = p;
    p += (size_t)a.DB * kBStage;
    s.kc = reinterpret_cast<float4 *>(p);
    p += (size_t)a.DK * kKStage;
    s.cc = reinterpret_cast<float *>(p);
    p += (size_t)a.DC * kCStage;
    s.raw = p;
    p += (size_t)a.DR * a.rawb;
    uint64_t *b = reinterpret_cast<uint64_t *>(p);
    s.raw_full = b; b += kMaxDR;
    s.raw_empty = b; b += kMaxDR;
    s.a_full = b; b += kMaxDA;
    s.a_empty = b; b += kMaxDA;
    s.b_full = b; b += kMaxDB;
    s.b_empty = b; b += kMaxDB;
    s.k_full = b; b += kMaxDK;
    s.k_empty = b; b += kMaxDK;
    s.c_full = b; b += kMaxDC;
    s.c_empty = b; b += kMaxDC;
    s.s_full = b; b += kSlots;
    s.s_empty = b; b += kSlots;
    s.done = b; b += 1;
    s.tmem_slot = reinterpret_cast<uint32_t *>(b);
    s.abort = reinterpret_cast<int *>(b) + 1;
    return s;
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

// ---------------------------------------------------------------- warp 3: unpack

// Four bits t0..t3 of t to the low bit of bytes 0..3 (the four partial products land on
// distinct bits, so nothing carries).
__device__ __forceinline__ uint32_t spread4(uint32_t t) {
    return ((t & 0xFu) * 0x00204081u) & 0x01010101u;
}

// The int8 operand of one 128-wide stage hs of a row's super-block (weights 128 hs .. 128 hs +
// 127 in their natural order; word 8 j + i holds weights 32 j + 4 i .. + 3 of block 4 hs + j).
//   Q4_K: sub-block 2p = low nibbles of qs[32p .. 32p + 32), 2p + 1 = their high nibbles.
//   Q5_K: the same plus the fifth bit, bit 2p (low) or 2p + 1 (high) of qh[l].
//   Q8_0: the quants of blocks 4 hs .. 4 hs + 3 as stored.
//   Q5_1: element l < 16 the low nibble of qs[l], l >= 16 the high nibble of qs[l - 16], the
//         fifth bit bit l of qh.
template <int FMT>
__device__ __forceinline__ void i8_stage(const uint8_t *rowp, int hs, uint32_t (&v)[32]) {
    if (FMT == MOE_FMT_Q4_K || FMT == MOE_FMT_Q5_K) {
        const uint8_t *qs = rowp + (FMT == MOE_FMT_Q5_K ? 48 : 16);
        uint32_t hw[8];
        if (FMT == MOE_FMT_Q5_K) {
            const uint4 *hp = reinterpret_cast<const uint4 *>(rowp + 16);
            const uint4 ha = hp[0], hb = hp[1];
            hw[0] = ha.x; hw[1] = ha.y; hw[2] = ha.z; hw[3] = ha.w;
            hw[4] = hb.x; hw[5] = hb.y; hw[6] = hb.z; hw[7] = hb.w;
        }
#pragma unroll
        for (int pp = 0; pp < 2; pp++) {
            const int p = 2 * hs + pp;
            const uint4 *qp = reinterpret_cast<const uint4 *>(qs + 32 * p);
            const uint4 qa = qp[0], qb = qp[1];
            const uint32_t x[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
            for (int w = 0; w < 8; w++) {
                uint32_t lo = x[w] & 0x0F0F0F0Fu, hi = (x[w] >> 4) & 0x0F0F0F0Fu;
                if (FMT == MOE_FMT_Q5_K) {
                    lo |= ((hw[w] >> (2 * p)) & 0x01010101u) << 4;
                    hi |= ((hw[w] >> (2 * p + 1)) & 0x01010101u) << 4;
                }
                v[16 * pp + w] = lo;
                v[16 * pp + 8 + w] = hi;
            }
        }
    } else if (FMT == MOE_FMT_Q8_0) {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int b = 4 * hs + j;
            const uint8_t *blk = rowp + 34 * b;
            if ((b & 1) == 0) {   // quants start 2 bytes past a word boundary
                const uint32_t *wp = reinterpret_cast<const uint32_t *>(blk);
                uint32_t wv[9];
#pragma unroll
                for (int i = 0; i < 9; i++) wv[i] = wp[i];
#pragma unroll
                for (int i = 0; i < 8; i++) v[8 * j + i] = __funnelshift_r(wv[i], wv[i + 1], 16);
            } else {
                const uint32_t *wp = reinterpret_cast<const uint32_t *>(blk + 2);
#pragma unroll
                for (int i = 0; i < 8; i++) v[8 * j + i] = wp[i];
            }
        }
    } else {   // Q5_1
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint2 *bp = reinterpret_cast<const uint2 *>(rowp + 24 * (4 * hs + j));
            const uint2 h = bp[0], qa = bp[1], qb = bp[2];
            const uint32_t qw[4] = {qa.x, qa.y, qb.x, qb.y};
#pragma unroll
            for (int w = 0; w < 4; w++) {
                v[8 * j + w] = (qw[w] & 0x0F0F0F0Fu) | (spread4(h.y >> (4 * w)) << 4);
                v[8 * j + 4 + w] =
                    ((qw[w] >> 4) & 0x0F0F0F0Fu) | (spread4(h.y >> (16 + 4 * w)) << 4);
            }
        }
    }
}

// The block constants of stage hs of a row's super-block: s_b and -wm_b of blocks 4 hs + j.
template <int FMT>
__device__ __forceinline__ void row_consts(const uint8_t *rowp, int hs, float (&s)[4],
                                           float (&nw)[4]) {
    if (FMT == MOE_FMT_Q4_K || FMT == MOE_FMT_Q5_K) {
        const uint4 hdr = *reinterpret_cast<const uint4 *>(rowp);
        const float d = half_bits_to_float(hdr.x), dmin = half_bits_to_float(hdr.x >> 16);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            int sc, mn;
            kq_scale_min(hdr.y, hdr.z, hdr.w, 4 * hs + j, sc, mn);
            s[j] = __fmul_rn(d, (float)sc);           // exact: 11 x 6 bits
            nw[j] = -__fmul_rn(dmin, (float)mn);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint8_t *blk = rowp + (FMT == MOE_FMT_Q8_0 ? 34 : 24) * (4 * hs + j);
            s[j] = half_bits_to_float(*reinterpret_cast<const uint16_t *>(blk));
            nw[j] = FMT == MOE_FMT_Q5_1
                        ? half_bits_to_float(*reinterpret_cast<const uint16_t *>(blk + 2))
                        : 0.0f;
        }
    }
}

template <int FMT>
__device__ __forceinline__ bool unpack_sb(const GemmArgs &a, const Smem &S, Ring &ra,
                                          const uint8_t *gb, const uint8_t *ub, uint32_t sbb) {
    const int u = threadIdx.x & 31;
#pragma unroll 1
    for (int hs = 0; hs < 2; hs++) {
        if (!waitw(a, S.abort, S.a_empty + ra.s, ra.ph ^ 1u)) return false;
        uint8_t *as = S.A + (size_t)ra.s * kAStage;
#pragma unroll 1
        for (int i = 0; i < 4; i++) {
            const int r = u + 32 * i;
            uint32_t v[32];
            i8_stage<FMT>(gb + (size_t)r * sbb, hs, v);
            store_row(as, r, v);
            i8_stage<FMT>(ub + (size_t)r * sbb, hs, v);
            store_row(as + kAtomA, r, v);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (u == 0) mbar_arrive(S.a_full + ra.s);
        ra.adv(1, kMaxDA);
    }
    return true;
}

__device__ void role_unpack(const GemmArgs &a, const Smem &S, int nj) {
    const int u = threadIdx.x & 31;
    Cursor cur;
    Ring rr, ra;
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
            const uint8_t *gb = S.raw + (size_t)rr.s * a.rawb;
            const uint8_t *ub = S.raw + (size_t)ru.s * a.rawb;
            bool ok;
            if (t.fmt == MOE_FMT_Q4_K) ok = unpack_sb<MOE_FMT_Q4_K>(a, S, ra, gb, ub, sbb);
            else if (t.fmt == MOE_FMT_Q5_K) ok = unpack_sb<MOE_FMT_Q5_K>(a, S, ra, gb, ub, sbb);
            else if (t.fmt == MOE_FMT_Q8_0) ok = unpack_sb<MOE_FMT_Q8_0>(a, S, ra, gb, ub, sbb);
            else ok = unpack_sb<MOE_FMT_Q5_1>(a, S, ra, gb, ub, sbb);
            if (!ok) return;
            __syncwarp();
            if (u == 0) {
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
    Ring ra, rb, rs;
    const uint32_t a_base = smem_u32(S.A), b_base = smem_u32(S.B);
    const int nst = a.H / 128;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const uint32_t idesc = instr_desc_i8(128, t.n_mma);
        for (int st = 0; st < nst; st++) {
            if (!wait1(a, S.abort, S.a_full + ra.s, ra.ph)) return;
            if (!wait1(a, S.abort, S.b_full + rb.s, rb.ph)) return;
            tc_fence_after();
            const uint64_t dAg = smem_desc(a_base + (uint32_t)ra.s * kAStage, 1024, 2);
            const uint64_t dAu = smem_desc(a_base + (uint32_t)ra.s * kAStage + kAtomA, 1024, 2);
            const uint64_t dB = smem_desc(b_base + (uint32_t)rb.s * kBStage, 1024, 2);
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {   // one 32-weight block per K-step (32 bytes)
                if (!wait1(a, S.abort, S.s_empty + rs.s, rs.ph ^ 1u)) return;
                tc_fence_after();
                const uint32_t d = tbase + (uint32_t)rs.s * 128;
                umma_i8(d, dAg + 2 * kk, dB + 2 * kk, idesc, 0u);
                umma_i8(d + 64, dAu + 2 * kk, dB + 2 * kk, idesc, 0u);
                umma_commit(S.s_full + rs.s);
                rs.adv(1, kSlots);
            }
            umma_commit(S.a_empty + ra.s);
            umma_commit(S.b_empty + rb.s);
            ra.adv(1, kMaxDA);
            rb.adv(1, a.DB);
        }
    }
}

// ---------------------------------------------------------------- warp 2: loader

__device__ __forceinline__ int column_token(const GemmArgs &a, const Tile &t, int n) {
    if (n >= t.n_valid) return -1;
    const int slot = t.slot_base + n;
    return t.shared ? slot - a.T * a.k : a.perm[slot] / a.k;
}

// The scales and block sums of blocks 4 st .. 4 st + 3 of token tok (0 for no token, so that
// padded columns add nothing).
struct ColConsts {
    uint2 d;
    float4 s;
};
__device__ __forceinline__ ColConsts col_consts(const GemmArgs &a, int tok, int st) {
    ColConsts c;
    c.d = make_uint2(0u, 0u);
    c.s = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (tok >= 0) {
        const int H32 = a.H / 32;
        c.d = *reinterpret_cast<const uint2 *>(a.xd + (size_t)tok * H32 + 4 * st);
        c.s = *reinterpret_cast<const float4 *>(a.xsum + (size_t)tok * H32 + 4 * st);
    }
    return c;
}

__device__ __forceinline__ void store_cols(float *cc, int n, const ColConsts &c) {
    cc[0 * kTN + n] = half_bits_to_float(c.d.x);
    cc[1 * kTN + n] = half_bits_to_float(c.d.x >> 16);
    cc[2 * kTN + n] = half_bits_to_float(c.d.y);
    cc[3 * kTN + n] = half_bits_to_float(c.d.y >> 16);
    cc[4 * kTN + 0 * kTN + n] = c.s.x;
    cc[4 * kTN + 1 * kTN + n] = c.s.y;
    cc[4 * kTN + 2 * kTN + n] = c.s.z;
    cc[4 * kTN + 3 * kTN + n] = c.s.w;
}

// The block constants of stage hs for rows lane + 32 i of gate and up, into a constant stage.
template <int FMT>
__device__ __forceinline__ void consts_stage(const uint8_t *gb, const uint8_t *ub, uint32_t sbb,
                                             int hs, float4 *kc, int lane) {
#pragma unroll 1
    for (int i = 0; i < 4; i++) {
        const int r = lane + 32 * i;
        float sg[4], ng[4], su[4], nu[4];
        row_consts<FMT>(gb + (size_t)r * sbb, hs, sg, ng);
        row_consts<FMT>(ub + (size_t)r * sbb, hs, su, nu);
#pragma unroll
        for (int j = 0; j < 4; j++) kc[j * 128 + r] = make_float4(sg[j], su[j], ng[j], nu[j]);
    }
}

__device__ void role_loader(const GemmArgs &a, const Smem &S, int nj) {
    const int lane = threadIdx.x & 31;
    const int c = lane & 7;                      // 16-byte chunk of a 128-byte row
    const int rg = lane >> 3;                    // rows rg + 4 j, j = 0..15
    Cursor cur;
    Ring rr, rb, rc, rk, ob;
    int npend = 0;
    bool ok = true;
    const int nsb = a.H / 256;
    for (int i = blockIdx.x; ok; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const uint32_t sbb = sb_bytes(t.fmt);
        const int tok0 = column_token(a, t, lane), tok1 = column_token(a, t, lane + 32);
        int src[16];                             // this lane's gather rows
#pragma unroll
        for (int j = 0; j < 16; j++) src[j] = column_token(a, t, rg + 4 * j);
        ColConsts n0 = col_consts(a, tok0, 0), n1 = col_consts(a, tok1, 0);
        ob = rb;
        auto signal_oldest = [&]() {
            if (lane == 0) mbar_arrive(S.b_full + ob.s);
            ob.adv(1, a.DB);
            npend--;
        };
        for (int sb = 0; sb < nsb && ok; sb++) {
            for (int hs = 0; hs < 2 && ok; hs++) {
                const int st = 2 * sb + hs;
                // the token rows of this 128-wide stage first: the oldest stage in flight is
                // signalled before the waits below on rings that the epilogue frees
                if (!(ok = waitw(a, S.abort, S.b_empty + rb.s, rb.ph ^ 1u))) break;
                uint8_t *bs = S.B + (size_t)rb.s * kBStage;
                const int8_t *col = a.xq + 128 * st + 16 * c;
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    const int n = rg + 4 * j;
                    if (src[j] >= 0) {
                        const uint32_t off = (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4);
                        cp_async16(bs + off, col + (size_t)src[j] * a.H);
                    }
                }
                cp_async_commit();
                npend++;
                rb.adv(1, a.DB);
                if (npend > a.lag) {
                    if (a.lag >= 3) cp_async_wait<3>();
                    else if (a.lag == 2) cp_async_wait<2>();
                    else cp_async_wait<1>();
                    fence_proxy_async_smem();
                    __syncwarp();
                    signal_oldest();
                }
                // the columns' scales and block sums (loaded one stage ahead)
                const ColConsts c0 = n0, c1 = n1;
                if (st + 1 < 2 * nsb) {
                    n0 = col_consts(a, tok0, st + 1);
                    n1 = col_consts(a, tok1, st + 1);
                }
                if (!(ok = waitw(a, S.abort, S.c_empty + rc.s, rc.ph ^ 1u))) break;
                float *cc = S.cc + (size_t)rc.s * (kCStage / 4);
                store_cols(cc, lane, c0);
                store_cols(cc, lane + 32, c1);
                __syncwarp();
                if (lane == 0) mbar_arrive(S.c_full + rc.s);
                rc.adv(1, a.DC);
                // the rows' block constants, from the packed rows
                Ring ru = rr;
                ru.adv(1, a.DR);
                if (hs == 0) {
                    if (!(ok = waitw(a, S.abort, S.raw_full + rr.s, rr.ph))) break;
                    if (!(ok = waitw(a, S.abort, S.raw_full + ru.s, ru.ph))) break;
                }
                if (!(ok = waitw(a, S.abort, S.k_empty + rk.s, rk.ph ^ 1u))) break;
                const uint8_t *gb = S.raw + (size_t)rr.s * a.rawb;
                const uint8_t *ub = S.raw + (size_t)ru.s * a.rawb;
                float4 *kc = S.kc + (size_t)rk.s * (kKStage / 16);
                if (t.fmt == MOE_FMT_Q4_K) consts_stage<MOE_FMT_Q4_K>(gb, ub, sbb, hs, kc, lane);
                else if (t.fmt == MOE_FMT_Q5_K) consts_stage<MOE_FMT_Q5_K>(gb, ub, sbb, hs, kc, lane);
                else if (t.fmt == MOE_FMT_Q8_0) consts_stage<MOE_FMT_Q8_0>(gb, ub, sbb, hs, kc, lane);
                else consts_stage<MOE_FMT_Q5_1>(gb, ub, sbb, hs, kc, lane);
                __syncwarp();
                if (lane == 0) mbar_arrive(S.k_full + rk.s);
                rk.adv(1, a.DK);
                if (hs == 1) {
                    if (lane == 0) {
                        mbar_arrive(S.raw_empty + rr.s);
                        mbar_arrive(S.raw_empty + ru.s);
                    }
                    rr.adv(2, a.DR);
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

// ---------------------------------------------------------------- warps 4-19: epilogue

// ---------------------------------------------------------------- the promotion (epilogue)

__device__ __forceinline__ uint64_t pk(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpk(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
// acc (this warp's 16 columns) += I * (s * xd) - wm * xs for one block, two columns per
// instruction.  The s32 value I converts to fp32 exactly (|I| < 2^24).
__device__ __forceinline__ void promote(uint64_t (&acc)[kEpiCols / 2], const uint32_t (&P)[16],
                                        float s, float nw, const float *xd, const float *xs) {
    const uint64_t s2 = pk(s, s), nw2 = pk(nw, nw);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const ulonglong2 xd4 = *reinterpret_cast<const ulonglong2 *>(xd + 2 * i);
        const ulonglong2 xs4 = *reinterpret_cast<const ulonglong2 *>(xs + 2 * i);
        const uint64_t f0 = pk(__int2float_rn((int)P[2 * i]), __int2float_rn((int)P[2 * i + 1]));
        const uint64_t f1 = pk(__int2float_rn((int)P[2 * i + 2]), __int2float_rn((int)P[2 * i + 3]));
        acc[i] = fma2(f0, mul2(s2, xd4.x), acc[i]);
        acc[i + 1] = fma2(f1, mul2(s2, xd4.y), acc[i + 1]);
        acc[i] = fma2(nw2, xs4.x, acc[i]);
        acc[i + 1] = fma2(nw2, xs4.y, acc[i + 1]);
    }
}

__device__ void role_epilogue(const GemmArgs &a, const Smem &S, int nj, uint32_t tbase) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;                  // tensor-memory lane quarter: rows 32q + lane
    const int ch = (warp - kEpiWarp0) >> 2;  // columns (tokens) 16 ch .. 16 ch + 15
    const int r = 32 * q + lane;
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    Cursor cur;
    Ring rk, rc, rs;
    const int nst = a.H / 128;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const bool active = kEpiCols * ch < t.n_mma;
        uint64_t ag[kEpiCols / 2], au[kEpiCols / 2];   // pairs of columns
#pragma unroll
        for (int j = 0; j < kEpiCols / 2; j++) ag[j] = au[j] = 0ull;
        for (int st = 0; st < nst; st++) {
            if (!waitw(a, S.abort, S.k_full + rk.s, rk.ph)) return;
            if (!waitw(a, S.abort, S.c_full + rc.s, rc.ph)) return;
            const float4 *kc = S.kc + (size_t)rk.s * (kKStage / 16);
            const float *cc = S.cc + (size_t)rc.s * (kCStage / 4);
#pragma unroll 1
            for (int j = 0; j < 4; j++) {
                if (!waitw(a, S.abort, S.s_full + rs.s, rs.ph)) return;
                tc_fence_after();
                // gate columns, then up; the slot is released once the second load has landed
                uint32_t P[16];
                float4 k4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                const float *xd = cc + j * kTN + kEpiCols * ch;
                const float *xs = cc + 4 * kTN + j * kTN + kEpiCols * ch;
                const uint32_t col = tbase + lane_addr + (uint32_t)rs.s * 128 + kEpiCols * ch;
                if (active) {
                    k4 = kc[j * 128 + r];
                    tmem_ld16(col, P);
                    tmem_ld_wait(P);
                    promote(ag, P, k4.x, k4.z, xd, xs);
                    tmem_ld16(col + 64, P);
                    tmem_ld_wait(P);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(S.s_empty + rs.s);
                rs.adv(1, kSlots);
                if (active) promote(au, P, k4.y, k4.w, xd, xs);
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(S.k_empty + rk.s);
                mbar_arrive(S.c_empty + rc.s);
            }
            rk.adv(1, a.DK);
            rc.adv(1, a.DC);
        }
        const int f = 128 * t.mt + r;
        const int nc = min(kEpiCols, t.n_valid - kEpiCols * ch);
        if (128 * t.mt + 32 * q < a.F) {   // the warp's 32 rows are one block of f, in range
#pragma unroll
            for (int j = 0; j < kEpiCols / 2; j++) {
                float g0, g1, u0, u1;
                unpk(ag[j], g0, g1);
                unpk(au[j], u0, u1);
                const int n = t.slot_base + kEpiCols * ch + 2 * j;
                if (2 * j < nc) quantize_h_lane(a, silu_mul(g0, u0), n, f);
                if (2 * j + 1 < nc) quantize_h_lane(a, silu_mul(g1, u1), n + 1, f);
            }
        }
    }
}

// ---------------------------------------------------------------- the kernel

__global__ void __launch_bounds__(kThreads, 1) k_gateup_i8(const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const Smem S = carve(base, a);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.DR; i++) {
            mbar_init(S.raw_full + i, 1);
            mbar_init(S.raw_empty + i, 2);   // the unpack warp and the loader
        }
        for (int i = 0; i < kMaxDA; i++) {
            mbar_init(S.a_full + i, 1);
            mbar_init(S.a_empty + i, 1);
        }
        for (int i = 0; i < a.DB; i++) {
            mbar_init(S.b_full + i, 1);
            mbar_init(S.b_empty + i, 1);
        }
        for (int i = 0; i < a.DK; i++) {
            mbar_init(S.k_full + i, 1);
            mbar_init(S.k_empty + i, kEpiWarps);
        }
        for (int i = 0; i < a.DC; i++) {
            mbar_init(S.c_full + i, 1);
            mbar_init(S.c_empty + i, kEpiWarps);
        }
        for (int i = 0; i < kSlots; i++) {
            mbar_init(S.s_full + i, 1);
            mbar_init(S.s_empty + i, kEpiWarps);
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
    } else if (warp == kLoadWarp) {
        role_loader(a, S, nj);
        __syncwarp();
    } else if (warp == kUnpackWarp) {
        role_unpack(a, S, nj);
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

// Ring depths that fit the shared memory: two operand stages; the deepest activation ring (four
// down to two 128-wide stages) with row-constant and column-constant rings as deep, that leaves
// room for three packed half-stages (one and a half super-blocks), else for two.  The loader
// signals an activation stage `lag` stages after issuing it, and before that it may wait for a
// constant slot that the epilogue frees only after the MMAs of the stage `depth` stages back: so
// lag <= the depth of both constant rings, or the loader waits for itself.
bool ring_plan(int fmt_mask, int &DB, int &DK, int &DC, int &DR) {
    const uint32_t rawb = raw_bytes(fmt_mask);
    for (int need = 3; need >= 2; need--) {
        for (DB = kMaxDB; DB >= 2; DB--) {
            DK = DB;
            DC = DB + 2 < kMaxDC ? DB + 2 : kMaxDC;
            const size_t fixed = smem_plan(DB, DK, DC, 0, rawb);
            if (fixed >= kSmemCap) continue;
            DR = (int)((kSmemCap - fixed) / rawb);
            if (DR > kMaxDR) DR = kMaxDR;
            if (DR >= need) return true;
        }
    }
    return false;
}

}  // namespace

size_t tc_gateup_i8_smem_bytes(int fmt_mask) {
    int DB, DK, DC, DR;
    if (!ring_plan(fmt_mask, DB, DK, DC, DR)) return (size_t)-1;
    return smem_plan(DB, DK, DC, DR, raw_bytes(fmt_mask));
}

cudaError_t launch_gateup_i8(const TcPhaseArgs &p, int grid, cudaStream_t st) {
    const FfnArgs &f = p.ffn;
    GemmArgs a{};
    a.wmaps = reinterpret_cast<const CUtensorMap *>(p.wmaps);
    a.experts = f.experts;
    a.jobs = f.jobs;
    a.njobs = f.njobs;
    a.perm = f.perm;
    a.w = f.w;
    a.xq = f.xq;
    a.xd = f.xd;
    a.xsum = f.xsum;
    a.T = f.T;
    a.k = f.k;
    a.H = f.H;
    a.F = f.F;
    a.hpad = f.hpad;
    a.mt_count = (f.F + 127) / 128;
    a.tn = kTN;
    if (!ring_plan(f.fmt_mask, a.DB, a.DK, a.DC, a.DR)) return cudaErrorInvalidValue;
    a.DA = kMaxDA;
    a.lag = a.DB - 1;   // <= DK and DC (ring_plan)
    a.rawb = raw_bytes(f.fmt_mask);
    a.hq = f.hq;
    a.hd = f.hd;
    a.hs = f.hs;
    a.hsum = f.hsum;
    a.h = p.keep_h ? f.h : nullptr;
    a.status = f.status;
    a.wait_ns = p.wait_ns;
    const size_t smem = smem_plan(a.DB, a.DK, a.DC, a.DR, a.rawb);
    if (grid <= 0) return cudaErrorInvalidDevice;
    cudaError_t err = ensure_smem(k_gateup_i8, smem);
    if (err != cudaSuccess) return err;
    if (std::getenv("MOE_DEBUG"))
        std::fprintf(stderr, "moe: k_gateup_i8 grid %d smem %zu rings B%d K%d C%d R%d rawb %u\n",
                     grid, smem, a.DB, a.DK, a.DC, a.DR, a.rawb);
    k_gateup_i8<<<grid, kThreads, smem, st>>>(a);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
