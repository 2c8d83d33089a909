// k_down_tc.cu -- a6 + a7 for large batches on the 5th-generation tensor cores (tcgen05):
// y = W_down h^ for every (expert, token) pair, weighted by the routing weight and scattered into
// out (or kept per slot for the deterministic combine); plus the operand preparation of both
// tensor-core phases and the tensor maps of the packed weights.
//
// One persistent kernel, one CTA per SM, over tiles of (expert job, up to 128 tokens, 256 output
// rows as two M = 128 operands whose accumulators sit side by side in tensor memory, double
// buffered).  Here the weights reach the tensor cores whole: unpack warps decode every packed
// weight into one fp16 value w = d*sc*q - dmin*m (Q4_K, Q5_K), d*q (Q8_0) or d*q + m (Q5_1),
// computed in fp16 (relative error ~2^-11 of the weight scale); the activation is Q8_1(h) of
// each slot, hd_j * q * 2^-e in fp16 (2^e from the slot's largest block scale, so that any finite
// h fits), rounded once.  One kind::f16 MMA chain with an fp32 accumulator runs over the whole
// contraction and the epilogue multiplies by 2^e.  Unlike the gate/up phase, nothing downstream
// re-quantizes y, so this rounding reaches the output as it is: ~1e-4 of the token's largest
// output, inside the layer's tolerance.
//
// Roles (512 threads, four warps per scheduler):
//   warp 0        TMA producer of the packed down rows (one super-block of 128 rows per load, L2
//                 prefetch two super-blocks ahead)
//   warp 1        tensor-memory allocation and the MMA issuer
//   warps 2-9     unpack: one thread per weight row of a 128-row operand, 64 weights per stage,
//                 written as the 128-byte-swizzled K-major fp16 operand
//   warps 10-11   activation loader: the tile's slot rows with 16-byte cp.async, and the
//                 tile's column table (token, routing weight, row scale)
//   warps 12-15   epilogue: weighted scatter into out (or y per slot)
// Both operands hold every group of 4 consecutive K positions in the order (0, 2, 1, 3): a
// contraction does not depend on the order of K, and this order lets one lop3 turn two packed
// nibbles into an fp16 pair.  Every hand-off is an mbarrier; every wait is bounded and a timeout
// ends the kernel with MOE_ERR_TIMEOUT after the copies in flight have landed.
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <vector>

#include "route_dev.cuh"
#include "tc_pipe.cuh"

namespace moe {

namespace {

using namespace ptx;
using namespace tcp;

constexpr int kTN = 128;                         // largest token count of a tile (MMA N)
constexpr int kUnpackWarps = 8;
constexpr int kLoadWarp0 = 2 + kUnpackWarps;     // 10
constexpr int kLoadWarps = 2;
constexpr int kEpiWarp0 = kLoadWarp0 + kLoadWarps;   // 12
constexpr int kEpiWarps = 4;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;   // 512
constexpr uint32_t kAtom = 16384;                // one operand atom: 128 rows x 64 fp16
constexpr uint32_t kAStage = 2 * kAtom;
constexpr uint32_t kBStage = kAtom;
constexpr int kMaxDA = 4, kMaxDB = 6, kMaxDR = 8;
constexpr uint32_t kTmemCols = 512;
constexpr size_t kSmemCap = 232448;              // opt-in dynamic shared memory per CTA, sm_100

// Per-tile column table, written by the loader, read by the epilogue.
struct TileInfo {
    int tok[kTN];
    float w[kTN];
    float scale[kTN];
    int pad[kTN];
};

struct Smem {
    uint8_t *A, *B, *raw;
    TileInfo *ti;
    uint64_t *raw_full, *raw_empty, *a_full, *a_empty, *b_full, *b_empty, *tm_full, *tm_empty,
        *ti_full, *ti_empty, *done;
    uint32_t *tmem_slot;
    int *abort;
};

__host__ __device__ inline size_t smem_plan(int DA, int DB, int DR, uint32_t rawb) {
    return 1024 + (size_t)DA * kAStage + (size_t)DB * kBStage + (size_t)DR * rawb +
           2 * sizeof(TileInfo) + 8 * (2 * kMaxDR + 2 * kMaxDA + 2 * kMaxDB + 9) + 16;
}

__device__ __forceinline__ Smem carve(uint8_t *base, const GemmArgs &a) {
    Smem s;
    uint8_t *p = base;
    s.A = p;
    p += (size_t)a.DA * kAStage;
    s.B = p;
    p += (size_t)a.DB * kBStage;
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
    s.tm_full = b; b += 2;
    s.tm_empty = b; b += 2;
    s.ti_full = b; b += 2;
    s.ti_empty = b; b += 2;
    s.done = b; b += 1;
    s.tmem_slot = reinterpret_cast<uint32_t *>(b);
    s.abort = reinterpret_cast<int *>(b) + 1;
    return s;
}

// ---------------------------------------------------------------- warp 0: weight producer

__device__ void role_producer(const GemmArgs &a, const Smem &S, int nj, Ring &rr, int &issued) {
    Cursor cur;
    const int nsb = (a.nst + 3) / 4;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const CUtensorMap *m = a.wmaps + (size_t)t.e * 3 + 2;
        const int y0 = t.mt * 256, y1 = y0 + 128;
        const uint32_t sbb = sb_bytes(t.fmt);
        const int xu = t.fmt == MOE_FMT_Q8_0 ? 136 : (int)sbb;   // Q8_0 maps count 16-bit units
        for (int sb = 0; sb < nsb; sb++) {
            if (sb + 2 < nsb) {
                tma_prefetch_2d(m, (sb + 2) * xu, y0);
                tma_prefetch_2d(m, (sb + 2) * xu, y1);
            }
            for (int hh = 0; hh < 2; hh++) {
                if (!wait1(a, S.abort, S.raw_empty + rr.s, rr.ph ^ 1u)) return;
                mbar_arrive_expect_tx(S.raw_full + rr.s, 128u * sbb);
                tma_load_2d(S.raw + (size_t)rr.s * a.rawb, m, sb * xu, hh ? y1 : y0,
                            S.raw_full + rr.s);
                issued++;
                rr.adv(1, a.DR);
            }
        }
    }
}

// ---------------------------------------------------------------- warps 2-9: unpack

// (1024 + q0, 1024 + q1) pair -> RN16(q * s) - m with s, -1024 s, m given as pairs.
__device__ __forceinline__ uint32_t kq_pair(uint32_t q1024, __half2 s, __half2 n1024s, __half2 m) {
    return h2u(__hsub2(__hfma2(u2h(q1024), s, n1024s), m));
}

// Whole weights of one 64-wide stage of a row as fp16, in the operand order (0, 2, 1, 3) inside
// every 4.  K-quants: stage st holds sub-blocks 2st (low nibbles of qs[32st .. 32st+32)) and 2st+1
// (high nibbles of the same bytes): positions 0..31 and 32..63 of the stage.
template <bool Q5>
__device__ __forceinline__ void kq_stage(const uint8_t *rowp, int st, uint32_t dscp, uint32_t dmmp,
                                         const uint32_t (&qh)[8], uint32_t (&v)[32]) {
    constexpr uint32_t kM = 0x000F000Fu, kE = 0x64006400u;
    const uint4 *qp = reinterpret_cast<const uint4 *>(rowp + (Q5 ? 48 : 16) + 32 * st);
    const uint4 qa = qp[0], qb = qp[1];
    const uint32_t qw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
    const __half2 sp = u2h(dscp), mp = u2h(dmmp);
    const __half2 s0 = __low2half2(sp), s1 = __high2half2(sp);
    const __half2 m0 = __low2half2(mp), m1 = __high2half2(mp);
    const __half2 k1024 = __float2half2_rn(-1024.0f);
    const __half2 n0 = __hmul2(s0, k1024), n1 = __hmul2(s1, k1024);
#pragma unroll
    for (int wi = 0; wi < 8; wi++) {
        const uint32_t x = qw[wi];
        uint32_t la = lop3_and_or(x, kM, kE), lb = lop3_and_or(x >> 8, kM, kE);
        uint32_t ha = lop3_and_or(x >> 4, kM, kE), hb = lop3_and_or(x >> 12, kM, kE);
        if (Q5) {   // fifth bits: bit 2st (low nibbles) and 2st+1 (high) of qh byte r
            const uint32_t t = qh[wi] >> (2 * st);
            la |= (t << 4) & 0x00100010u;
            lb |= (t >> 4) & 0x00100010u;
            ha |= (t << 3) & 0x00100010u;
            hb |= (t >> 5) & 0x00100010u;
        }
        // word wi covers positions 4wi..4wi+3 of each sub-block: chunk wi/2, half wi%2
        v[2 * wi] = kq_pair(la, s0, n0, m0);
        v[2 * wi + 1] = kq_pair(lb, s0, n0, m0);
        v[16 + 2 * wi] = kq_pair(ha, s1, n1, m1);
        v[16 + 2 * wi + 1] = kq_pair(hb, s1, n1, m1);
    }
}

// Q8_0: stage st holds blocks 2st and 2st+1 (34 bytes each; odd blocks' quants are 4-byte
// aligned, even blocks' start 2 bytes past a word boundary).
__device__ __forceinline__ void q80_stage(const uint8_t *rowp, int st, uint32_t (&v)[32]) {
    const __half2 k1152 = __float2half2_rn(1152.0f);
#pragma unroll
    for (int bb = 0; bb < 2; bb++) {
        const int b = 2 * st + bb;
        const uint8_t *blk = rowp + 34 * b;
        const __half dh = *reinterpret_cast<const __half *>(blk);
        const __half2 d2 = __half2half2(dh);
        uint32_t q[8];
        if (bb == 0) {   // words at blk (aligned): bytes 2.. of the first
            const uint32_t *wp = reinterpret_cast<const uint32_t *>(blk);
            uint32_t w[9];
#pragma unroll
            for (int i = 0; i < 9; i++) w[i] = wp[i];
#pragma unroll
            for (int i = 0; i < 8; i++) q[i] = __funnelshift_r(w[i], w[i + 1], 16);
        } else {
            const uint32_t *wp = reinterpret_cast<const uint32_t *>(blk + 2);
#pragma unroll
            for (int i = 0; i < 8; i++) q[i] = wp[i];
        }
#pragma unroll
        for (int i = 0; i < 8; i++) {
            // bytes b -> fp16 (1024 + (b ^ 0x80)) - 1152 = b (exact), times d
            const uint32_t x = q[i] ^ 0x80808080u;
            const __half2 a = __hsub2(u2h(prmt(x, 0x64646464u, 0x4240u)), k1152);
            const __half2 c = __hsub2(u2h(prmt(x, 0x64646464u, 0x4341u)), k1152);
            v[16 * bb + 2 * i] = h2u(__hmul2(a, d2));
            v[16 * bb + 2 * i + 1] = h2u(__hmul2(c, d2));
        }
    }
}

// Q5_1: stage st holds blocks 2st and 2st+1 (24 bytes each, 8-byte aligned).
__device__ __forceinline__ void q51_stage(const uint8_t *rowp, int st, uint32_t (&v)[32]) {
    constexpr uint32_t kM = 0x000F000Fu, kE = 0x64006400u;
    const __half2 k1024 = __float2half2_rn(-1024.0f);
#pragma unroll
    for (int bb = 0; bb < 2; bb++) {
        const uint2 *bp = reinterpret_cast<const uint2 *>(rowp + 24 * (2 * st + bb));
        const uint2 h = bp[0], qa = bp[1], qb = bp[2];
        const __half2 d2 = __half2half2(__ushort_as_half((unsigned short)(h.x & 0xFFFFu)));
        const __half2 m2 = __half2half2(__ushort_as_half((unsigned short)(h.x >> 16)));
        const __half2 n2 = __hmul2(d2, k1024);
        const uint32_t qw[4] = {qa.x, qa.y, qb.x, qb.y};
#pragma unroll
        for (int wi = 0; wi < 8; wi++) {
            // elements 4wi..4wi+3: n < 16 low nibbles of qs[n], n >= 16 high nibbles of qs[n-16]
            const uint32_t x = wi < 4 ? qw[wi] : qw[wi - 4] >> 4;
            const uint32_t t = h.y >> (4 * wi);
            const uint32_t pa = lop3_and_or(x, kM, kE) | (((t & 5u) * 0x40010u) & 0x00100010u);
            const uint32_t pb = lop3_and_or(x >> 8, kM, kE) | (((t & 10u) * 0x20008u) & 0x00100010u);
            v[16 * bb + 2 * wi] = h2u(__hadd2(__hfma2(u2h(pa), d2, n2), m2));
            v[16 * bb + 2 * wi + 1] = h2u(__hadd2(__hfma2(u2h(pb), d2, n2), m2));
        }
    }
}

template <int FMT>
__device__ __forceinline__ bool unpack_superblock(const GemmArgs &a, const Smem &S, Ring &ra,
                                                  const uint8_t *rowp, int nst_sb, int half,
                                                  int r) {
    const int lane = threadIdx.x & 31;
    uint32_t dscp[4] = {0, 0, 0, 0}, dmmp[4] = {0, 0, 0, 0};
    uint32_t qh[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (FMT == MOE_FMT_Q4_K || FMT == MOE_FMT_Q5_K) {
        const uint4 hdr = *reinterpret_cast<const uint4 *>(rowp);
        const float d = half_bits_to_float(hdr.x), dmin = half_bits_to_float(hdr.x >> 16);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            int sc0, mn0, sc1, mn1;
            kq_scale_min(hdr.y, hdr.z, hdr.w, j, sc0, mn0);
            kq_scale_min(hdr.y, hdr.z, hdr.w, j + 1, sc1, mn1);
            dscp[j / 2] = h2u(__floats2half2_rn(d * (float)sc0, d * (float)sc1));
            dmmp[j / 2] = h2u(__floats2half2_rn(dmin * (float)mn0, dmin * (float)mn1));
        }
        if (FMT == MOE_FMT_Q5_K) {
            const uint4 *hp = reinterpret_cast<const uint4 *>(rowp + 16);
            const uint4 ha = hp[0], hb = hp[1];
            qh[0] = ha.x; qh[1] = ha.y; qh[2] = ha.z; qh[3] = ha.w;
            qh[4] = hb.x; qh[5] = hb.y; qh[6] = hb.z; qh[7] = hb.w;
        }
    }
#pragma unroll 1
    for (int st = 0; st < nst_sb; st++) {
        if (!waitw(a, S.abort, S.a_empty + ra.s, ra.ph ^ 1u)) return false;
        uint32_t v[32];
        if (FMT == MOE_FMT_Q4_K || FMT == MOE_FMT_Q5_K) {
            const uint32_t sp = st == 0 ? dscp[0] : st == 1 ? dscp[1] : st == 2 ? dscp[2] : dscp[3];
            const uint32_t mp = st == 0 ? dmmp[0] : st == 1 ? dmmp[1] : st == 2 ? dmmp[2] : dmmp[3];
            kq_stage<FMT == MOE_FMT_Q5_K>(rowp, st, sp, mp, qh, v);
        } else if (FMT == MOE_FMT_Q8_0) {
            q80_stage(rowp, st, v);
        } else {
            q51_stage(rowp, st, v);
        }
        store_row(S.A + (size_t)ra.s * kAStage + half * kAtom, r, v);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(S.a_full + ra.s);
        ra.adv(1, a.DA);
    }
    return true;
}


__device__ void role_unpack(const GemmArgs &a, const Smem &S, int nj) {
    const int u = threadIdx.x - 64;          // 0..255
    const int half = u >> 7, r = u & 127;    // the two 128-row operands, row
    const int lane = threadIdx.x & 31;
    Cursor cur;
    Ring rr, ra;
    rr.adv(half, a.DR);                      // this half's packed stages: every other one
    const int nsb = (a.nst + 3) / 4;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const uint32_t sbb = sb_bytes(t.fmt);
        for (int sb = 0; sb < nsb; sb++) {
            const int nst_sb = min(4, a.nst - 4 * sb);
            if (!waitw(a, S.abort, S.raw_full + rr.s, rr.ph)) return;
            const uint8_t *rowp = S.raw + (size_t)rr.s * a.rawb + (size_t)r * sbb;
            bool ok;
            if (t.fmt == MOE_FMT_Q4_K)
                ok = unpack_superblock<MOE_FMT_Q4_K>(a, S, ra, rowp, nst_sb, half, r);
            else if (t.fmt == MOE_FMT_Q5_K)
                ok = unpack_superblock<MOE_FMT_Q5_K>(a, S, ra, rowp, nst_sb, half, r);
            else if (t.fmt == MOE_FMT_Q8_0)
                ok = unpack_superblock<MOE_FMT_Q8_0>(a, S, ra, rowp, nst_sb, half, r);
            else
                ok = unpack_superblock<MOE_FMT_Q5_1>(a, S, ra, rowp, nst_sb, half, r);
            if (!ok) return;
            __syncwarp();
            if (lane == 0) mbar_arrive(S.raw_empty + rr.s);
            rr.adv(2, a.DR);
        }
    }
}

// ---------------------------------------------------------------- warp 1: MMA issuer

__device__ void role_mma(const GemmArgs &a, const Smem &S, int nj, uint32_t tbase) {
    Cursor cur;
    Ring ra, rb, rt;
    const uint32_t a_base = smem_u32(S.A), b_base = smem_u32(S.B);
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        const uint32_t idesc = instr_desc(0, 128, t.n_mma);
        if (!wait1(a, S.abort, S.tm_empty + rt.s, rt.ph ^ 1u)) return;
        tc_fence_after();
        const uint32_t d0 = tbase + (uint32_t)rt.s * 256, d1 = d0 + 128;
        for (int g = 0; g < a.nst; g++) {
            if (!wait1(a, S.abort, S.a_full + ra.s, ra.ph)) return;
            if (!wait1(a, S.abort, S.b_full + rb.s, rb.ph)) return;
            tc_fence_after();
            const uint64_t dA0 = smem_desc(a_base + (uint32_t)ra.s * kAStage, 1024, 2);
            const uint64_t dA1 = smem_desc(a_base + (uint32_t)ra.s * kAStage + kAtom, 1024, 2);
            const uint64_t dB = smem_desc(b_base + (uint32_t)rb.s * kBStage, 1024, 2);
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {   // K = 16 per instruction: +32 bytes in the atom
                const uint32_t acc = (g | kk) ? 1u : 0u;
                umma_f16(d0, dA0 + 2 * kk, dB + 2 * kk, idesc, acc);
                umma_f16(d1, dA1 + 2 * kk, dB + 2 * kk, idesc, acc);
            }
            umma_commit(S.a_empty + ra.s);
            umma_commit(S.b_empty + rb.s);
            ra.adv(1, a.DA);
            rb.adv(1, a.DB);
        }
        umma_commit(S.tm_full + rt.s);
        rt.adv(1, 2);
    }
}

// ---------------------------------------------------------------- warps 10-11: activation loader

__device__ void role_loader(const GemmArgs &a, const Smem &S, int nj) {
    const int lt = threadIdx.x - kLoadWarp0 * 32;   // 0..63
    const int lane = lt & 31, wl = lt >> 5;
    const int c = lane & 7;                        // 16-byte chunk of a 128-byte row
    const int rg = 4 * wl + (lane >> 3);           // rows rg + 8 j, j = 0..15
    Cursor cur;
    Ring rb, rt, ob;                               // ob: oldest stage issued, not yet signalled
    int npend = 0;
    bool ok = true;
    for (int i = blockIdx.x; ok; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        if (!(ok = waitw(a, S.abort, S.ti_empty + rt.s, rt.ph ^ 1u))) break;
        TileInfo &ti = S.ti[rt.s];
#pragma unroll
        for (int h = 0; h < 2; h++) {   // columns lt and lt + 64 of the epilogue's table
            const int n = lt + 64 * h;
            if (n < t.n_valid) {
                const int slot = t.slot_base + n;
                int tok;
                float wt;
                if (t.shared) {
                    tok = slot - a.T * a.k;
                    wt = a.gate ? a.gate[tok] : 1.0f;
                } else {
                    const int p = a.perm[slot];
                    tok = p / a.k;
                    wt = a.w[p];
                }
                ti.tok[n] = tok;
                ti.w[n] = wt;
                ti.scale[n] = a.act_scale[slot];
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(S.ti_full + rt.s);
        rt.adv(1, 2);
        for (int g = 0; g < a.nst; g++) {
            if (!(ok = waitw(a, S.abort, S.b_empty + rb.s, rb.ph ^ 1u))) break;
            uint8_t *bs = S.B + (size_t)rb.s * kBStage;
            const __half *col = a.act + (size_t)t.slot_base * a.act_pitch + 64 * g + 8 * c;
#pragma unroll
            for (int j = 0; j < 16; j++) {
                const int n = rg + 8 * j;
                if (n < t.n_valid)
                    cp_async16(bs + (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4),
                               col + (size_t)n * a.act_pitch);
            }
            cp_async_commit();
            if (npend++ == 0) ob = rb;
            rb.adv(1, a.DB);
            if (npend > a.lag) {
                if (a.lag >= 3) cp_async_wait<3>();
                else cp_async_wait<2>();
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(S.b_full + ob.s);
                ob.adv(1, a.DB);
                npend--;
            }
        }
        // the tile's last stages: land them now rather than after the next tile's set-up
        cp_async_wait<0>();
        fence_proxy_async_smem();
        __syncwarp();
        for (; npend > 0; npend--) {
            if (lane == 0) mbar_arrive(S.b_full + ob.s);
            ob.adv(1, a.DB);
        }
    }
    cp_async_wait<0>();
}

// ---------------------------------------------------------------- warps 12-15: epilogue

__device__ void role_epilogue(const GemmArgs &a, const Smem &S, int nj, uint32_t tbase) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;                  // tensor-memory lane quarter of this warp
    Cursor cur;
    Ring rt;
    for (int i = blockIdx.x;; i += gridDim.x) {
        Tile t;
        if (!tile_at(a, nj, cur, i, t)) break;
        if (!waitw(a, S.abort, S.tm_full + rt.s, rt.ph)) return;
        if (!waitw(a, S.abort, S.ti_full + rt.s, rt.ph)) return;
        tc_fence_after();
        const TileInfo &ti = S.ti[rt.s];
        const uint32_t tcol = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)rt.s * 256;
        const int row = 256 * t.mt + 32 * q + lane;   // output rows row, row + 128
#pragma unroll 1
        for (int c0 = 0; c0 < t.n_valid; c0 += 32) {
            uint32_t r0[32], r1[32];
            tmem_ld32(tcol + c0, r0);
            tmem_ld32(tcol + 128 + c0, r1);
            tmem_ld_wait(r0);
            reg_tie(r1);
            const int nc = min(32, t.n_valid - c0);
#pragma unroll
            for (int j = 0; j < 32; j++) {
                if (j < nc) {
                    const int n = c0 + j;
                    const float s = ti.scale[n];
                    const float y0 = __uint_as_float(r0[j]) * s;
                    const float y1 = __uint_as_float(r1[j]) * s;
                    if (a.y) {
                        float *yr = a.y + (size_t)(t.slot_base + n) * a.H;
                        yr[row] = y0;
                        yr[row + 128] = y1;
                    } else {
                        const float wv = ti.w[n];
                        float *orow = a.out + (size_t)ti.tok[n] * a.H;
                        atomicAdd(orow + row, wv * y0);
                        atomicAdd(orow + row + 128, wv * y1);
                    }
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(S.tm_empty + rt.s);
            mbar_arrive(S.ti_empty + rt.s);
        }
        rt.adv(1, 2);
    }
}

// ---------------------------------------------------------------- the kernel

__global__ void __launch_bounds__(kThreads, 1) k_down_tc(const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const Smem S = carve(base, a);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.DR; i++) {
            mbar_init(S.raw_full + i, 1);
            mbar_init(S.raw_empty + i, kUnpackWarps / 2);
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

// ---------------------------------------------------------------- operand preparation kernels

// Eight Q8_1 values (int8 q, fp32 scale s = xd * 2^-e) as fp16 q * s rounded once (and, with lo,
// the remainder q * s - hi, exact: q * s has at most 19 significant bits), in the operand order
// (0, 2, 1, 3) inside every 4.
__device__ __forceinline__ uint4 act8(uint2 qv, float s, uint4 *lo) {
    const int8_t *b = reinterpret_cast<const int8_t *>(&qv);
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; i++) v[i] = (float)b[i] * s;   // exact: 8 x 11 significant bits
    const __half2 h0 = __floats2half2_rn(v[0], v[2]), h1 = __floats2half2_rn(v[1], v[3]);
    const __half2 h2 = __floats2half2_rn(v[4], v[6]), h3 = __floats2half2_rn(v[5], v[7]);
    if (lo) {
        const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
        const float2 f2 = __half22float2(h2), f3 = __half22float2(h3);
        lo->x = h2u(__floats2half2_rn(v[0] - f0.x, v[2] - f0.y));
        lo->y = h2u(__floats2half2_rn(v[1] - f1.x, v[3] - f1.y));
        lo->z = h2u(__floats2half2_rn(v[4] - f2.x, v[6] - f2.y));
        lo->w = h2u(__floats2half2_rn(v[5] - f3.x, v[7] - f3.y));
    }
    return make_uint4(h2u(h0), h2u(h1), h2u(h2), h2u(h3));
}

// a1 for the tensor-core path: one warp per token.  Q8_1 of the row exactly as k_quantize (same
// block routine); then, with 2^e the row's power-of-two scale, the gate/up operand x^ * 2^-e as
// fp16 hi + lo planes (exact), and each block's sum xd * sum(q) * 2^-e as tf32 hi + lo.
__global__ void __launch_bounds__(256) k_quant_rows(const float *__restrict__ x, int T, int H,
                                                    int8_t *xq, uint16_t *xd, uint16_t *xs,
                                                    float *xsum, __half *xh, __half *xl,
                                                    float *xsh, float *xsl, float *xscale,
                                                    uint32_t *status) {
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    const int nb = H / 32;
    const int sub = lane & 7, grp = lane >> 3;
    const float *xr = x + (size_t)t * H;
    int8_t *qr = xq + (size_t)t * H;
    uint16_t *dr = xd + (size_t)t * nb;
    float *sr = xsum + (size_t)t * nb;
    for (int b0 = 0; b0 < nb; b0 += 4) {
        const int b = b0 + grp;
        const bool act = b < nb;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (act) v = __ldg(reinterpret_cast<const float4 *>(xr + 32 * b) + sub);
        const int bb = act ? b : 0;
        q8_1_block8(v, act, sub, qr + 32 * bb, dr + bb, xs + (size_t)t * nb + bb, sr + bb, status);
    }
    __syncwarp();
    float m = 0.0f;
    for (int j = lane; j < nb; j += 32) m = fmaxf(m, half_bits_to_float(dr[j]));
    m = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m)));
    float inv;
    const float sc = row_scale(m, &inv);
    if (lane == 0) xscale[t] = sc;
    for (int j = lane; j < nb; j += 32) {
        const float v = sr[j] * inv;   // exact (a power of two)
        const float hi = tf32_round(v);
        xsh[(size_t)t * nb + j] = hi;
        xsl[(size_t)t * nb + j] = tf32_round(v - hi);
    }
    __half *hr = xh + (size_t)t * H, *lr = xl + (size_t)t * H;
    for (int c = lane; c < H / 8; c += 32) {
        const uint2 qv = *reinterpret_cast<const uint2 *>(qr + 8 * c);
        const float s = half_bits_to_float(dr[c / 4]) * inv;
        uint4 lo;
        *reinterpret_cast<uint4 *>(hr + 8 * c) = act8(qv, s, &lo);
        *reinterpret_cast<uint4 *>(lr + 8 * c) = lo;
    }
}

// The down phase's operand: h^ = hd_j * q * 2^-e per slot (fp16, rounded once), zero from F to
// Kd, and 2^e.  One warp per slot.
__global__ void __launch_bounds__(256) k_h_rows(const int8_t *__restrict__ hq,
                                                const uint16_t *__restrict__ hd, int slots, int F,
                                                int hpad, int Kd, __half *hh, float *hscale) {
    const int s = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (s >= slots) return;
    const int hb = hpad / 32, nb = F / 32;
    const uint16_t *dr = hd + (size_t)s * hb;
    float m = 0.0f;
    for (int j = lane; j < nb; j += 32) m = fmaxf(m, half_bits_to_float(dr[j]));
    m = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m)));
    float inv;
    const float sc = row_scale(m, &inv);
    if (lane == 0) hscale[s] = sc;
    const int8_t *qr = hq + (size_t)s * hpad;
    __half *out = hh + (size_t)s * Kd;
    for (int c = lane; c < Kd / 8; c += 32) {
        uint4 o = make_uint4(0, 0, 0, 0);
        if (8 * c < F) {
            const uint2 qv = *reinterpret_cast<const uint2 *>(qr + 8 * c);
            o = act8(qv, half_bits_to_float(dr[c / 4]) * inv, nullptr);
        }
        *reinterpret_cast<uint4 *>(out + 8 * c) = o;
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

bool encode_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t dim0,
               uint64_t dim1, uint64_t stride_bytes, uint32_t box0, uint32_t box1) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {dim0, dim1};
    const cuuint64_t strides[1] = {stride_bytes};
    const cuuint32_t box[2] = {box0, box1};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

uint32_t raw_bytes(int fmt_mask) {
    uint32_t sbb_max = 0;
    for (int fm = 0; fm <= MOE_FMT_Q5_1; fm++)
        if (fmt_mask & (1 << fm)) sbb_max = sbb_max > sb_bytes(fm) ? sbb_max : sb_bytes(fm);
    return ((128u * sbb_max) + 1023u) & ~1023u;
}

// Ring depths that fit the shared memory: two unpacked-weight stages, four or three activation
// stages, and as many packed stages (at least three) as the rest allows.
bool ring_plan(int fmt_mask, int &DA, int &DB, int &DR) {
    const uint32_t rawb = raw_bytes(fmt_mask);
    DA = 2;
    for (DB = 4; DB >= 3; DB--) {
        const size_t fixed = smem_plan(DA, DB, 0, rawb);
        if (fixed >= kSmemCap) continue;
        DR = (int)((kSmemCap - fixed) / rawb);
        if (DR > kMaxDR) DR = kMaxDR;
        if (DR >= 3) return true;
    }
    return false;
}

}  // namespace

// Tensor maps of every expert's three packed matrices, as boxes of one super-block (256
// weights) x 128 rows.  Returns false when a map cannot be encoded (the caller then keeps the
// CUDA-core kernels for large batches).
bool tc_build_weight_maps(const uint8_t *d_base, const moe_expert_desc *descs, int n, int H,
                          int F, std::vector<uint8_t> &out) {
    if (H % 256 != 0 || F % 64 != 0) return false;
    out.assign((size_t)n * 3 * sizeof(CUtensorMap), 0);
    CUtensorMap *maps = reinterpret_cast<CUtensorMap *>(out.data());
    for (int e = 0; e < n; e++) {
        const moe_expert_desc &d = descs[e];
        if (d.fmt == MOE_FMT_Q6_K) return false;   // no exact fp16 operand form
        for (int t = 0; t < 3; t++) {
            const int rows = t < 2 ? F : H;
            const int width = t < 2 ? H : F;
            const void *base = d_base + d.off[t];
            bool ok;
            if (d.fmt == MOE_FMT_Q8_0) {
                const uint64_t nb = (uint64_t)((width + 31) / 32);
                ok = encode_2d(&maps[e * 3 + t], CU_TENSOR_MAP_DATA_TYPE_UINT16, base, nb * 17,
                               (uint64_t)rows, d.stride[t], 136, 128);
            } else if (d.fmt == MOE_FMT_Q5_1) {
                const uint64_t nb = (uint64_t)((width + 31) / 32);
                ok = encode_2d(&maps[e * 3 + t], CU_TENSOR_MAP_DATA_TYPE_UINT8, base, nb * 24,
                               (uint64_t)rows, d.stride[t], 192, 128);
            } else {
                const uint32_t sbb = sb_bytes(d.fmt);
                const uint64_t nsb = (uint64_t)((width + 255) / 256);
                ok = encode_2d(&maps[e * 3 + t], CU_TENSOR_MAP_DATA_TYPE_UINT8, base, nsb * sbb,
                               (uint64_t)rows, d.stride[t], sbb, 128);
            }
            if (!ok) return false;
        }
    }
    return true;
}


size_t tc_smem_bytes(int fmt_mask) {
    int DA, DB, DR;
    if (!ring_plan(fmt_mask, DA, DB, DR)) return (size_t)-1;
    const size_t down = smem_plan(DA, DB, DR, raw_bytes(fmt_mask));
    const size_t gu = tc_gateup_smem_bytes(fmt_mask);
    const size_t gi = tc_gateup_i8_smem_bytes(fmt_mask);
    if (gu == (size_t)-1 || gi == (size_t)-1) return (size_t)-1;
    const size_t m = down > gu ? down : gu;
    return m > gi ? m : gi;
}

// The tensor-core phases of one layer: gate/up (k_gateup_tc.cu), then the down operand and the
// down projection.
cudaError_t launch_gemm_tc(const TcPhaseArgs &p, cudaStream_t st) {
    const int grid = sm_count();
    if (grid <= 0) return cudaErrorInvalidDevice;
    if (p.phase == 0) return p.i8 ? launch_gateup_i8(p, grid, st) : launch_gateup_tc(p, grid, st);
    const FfnArgs &f = p.ffn;
    GemmArgs a{};
    a.wmaps = reinterpret_cast<const CUtensorMap *>(p.wmaps);
    a.experts = f.experts;
    a.jobs = f.jobs;
    a.njobs = f.njobs;
    a.perm = f.perm;
    a.w = f.w;
    a.act = p.hh;
    a.act_scale = p.hscale;
    a.act_pitch = p.Kd;
    a.T = f.T;
    a.k = f.k;
    a.H = f.H;
    a.F = f.F;
    a.hpad = f.hpad;
    a.nst = p.Kd / 64;
    a.mt_count = f.H / 256;
    a.tn = kTN;
    if (!ring_plan(f.fmt_mask, a.DA, a.DB, a.DR)) return cudaErrorInvalidValue;
    a.lag = a.DB - 1;
    a.rawb = raw_bytes(f.fmt_mask);
    a.out = f.out;
    a.gate = f.gate;
    a.y = f.y;
    a.status = f.status;
    a.wait_ns = p.wait_ns;
    const size_t smem = smem_plan(a.DA, a.DB, a.DR, a.rawb);
    cudaError_t err = ensure_smem(k_down_tc, smem);
    if (err != cudaSuccess) return err;
    if (std::getenv("MOE_DEBUG"))
        std::fprintf(stderr, "moe: k_down_tc grid %d smem %zu rings %d/%d/%d rawb %u nst %d\n",
                     grid, smem, a.DA, a.DB, a.DR, a.rawb, a.nst);
    k_down_tc<<<grid, kThreads, smem, st>>>(a);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_quant_rows(const float *x, int T, int H, int8_t *xq, uint16_t *xd,
                              uint16_t *xs, float *xsum, __half *xh, __half *xl, float *xsh,
                              float *xsl, float *xscale, uint32_t *status, cudaStream_t st) {
    if (T <= 0) return cudaSuccess;
    k_quant_rows<<<(T + 7) / 8, 256, 0, st>>>(x, T, H, xq, xd, xs, xsum, xh, xl, xsh, xsl, xscale,
                                              status);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_h_rows(const int8_t *hq, const uint16_t *hd, int slots, int F, int hpad, int Kd,
                          __half *hh, float *hscale, cudaStream_t st) {
    if (slots <= 0) return cudaSuccess;
    k_h_rows<<<(slots + 7) / 8, 256, 0, st>>>(hq, hd, slots, F, hpad, Kd, hh, hscale);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
