// dot.cuh -- per-lane partial dot products of packed K-quant / Q8_0 / Q5_1 rows with Q8_1
// activations, and the small warp-level helpers the FFN kernels share.
//
// For a sub-block of 32 weights w = d*sc*q - dmin*m and Q8_1 activations xd*qx, the dot is
//   d*sc*xd*sum(q*qx) - dmin*m*(xd*sum qx)
// where xd*sum(qx) is kept exactly in fp32 per activation block ("xsum").  A Q5_1 block
// (w = d*q + m) is the same with sc = 1 and the offset added: d*xd*sum(q*qx) + m*(xd*sum qx).
#pragma once

#include "moe_internal.cuh"

namespace moe {

constexpr unsigned kFullMask = 0xffffffffu;

__device__ __forceinline__ uint4 ld_stream16(const uint8_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ld_stream8(const uint8_t *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream_u32(const uint8_t *p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream_u16(const uint8_t *p) {
    unsigned short v;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(kFullMask, v, o);
    return v;
}

// Activations of one row set, Q8_1 SoA: q [K], d (fp32) [K/32], exact xd*sum(q) [K/32].
struct ActRow {
    const int8_t *q;
    const float *d;
    const float *s;
};

// ------------------------------------------------------------------ per-lane partial dots

// Unpacked 4-bit (Q4_K) or 5-bit (Q5_K) quants of lane part j of one super-block.
struct KqLane {
    uint32_t lo[4], hi[4];
    float dl, dh, ml, mh;   // d*sc and dmin*m of sub-blocks 2c and 2c+1
};

template <int FMT>
__device__ __forceinline__ KqLane kq_unpack(uint4 hdr, uint4 qv, uint4 qh, int j) {
    const int c = j >> 1;
    KqLane r;
    const float d = half_bits_to_float(hdr.x);
    const float dmin = half_bits_to_float(hdr.x >> 16);
    int scl, ml, sch, mh;
    kq_scale_min(hdr.y, hdr.z, hdr.w, 2 * c, scl, ml);
    kq_scale_min(hdr.y, hdr.z, hdr.w, 2 * c + 1, sch, mh);
    r.dl = d * (float)scl;
    r.dh = d * (float)sch;
    r.ml = dmin * (float)ml;
    r.mh = dmin * (float)mh;
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
    const uint32_t hw[4] = {qh.x, qh.y, qh.z, qh.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        r.lo[i] = qw[i] & 0x0F0F0F0Fu;
        r.hi[i] = (qw[i] >> 4) & 0x0F0F0F0Fu;
        if (FMT == MOE_FMT_Q5_K) {
            r.lo[i] |= ((hw[i] >> (2 * c)) & 0x01010101u) << 4;
            r.hi[i] |= ((hw[i] >> (2 * c + 1)) & 0x01010101u) << 4;
        }
    }
    return r;
}

// Lane's share of sum_k w_k * xhat_k: xa / xb are the 16 activation bytes matching the low /
// high nibbles, xd* the Q8_1 scales and xs* the exact xd*sum(q) of blocks 2c and 2c+1.  The
// min term of a whole sub-block is added by the hh == 0 lane only.
__device__ __forceinline__ float kq_dot(const KqLane &w, int hh, int4 xa, int4 xb, float xdl,
                                        float xdh, float xsl, float xsh) {
    int il = __dp4a((int)w.lo[0], xa.x, 0);
    il = __dp4a((int)w.lo[1], xa.y, il);
    il = __dp4a((int)w.lo[2], xa.z, il);
    il = __dp4a((int)w.lo[3], xa.w, il);
    int ih = __dp4a((int)w.hi[0], xb.x, 0);
    ih = __dp4a((int)w.hi[1], xb.y, ih);
    ih = __dp4a((int)w.hi[2], xb.z, ih);
    ih = __dp4a((int)w.hi[3], xb.w, ih);
    float r = w.dl * xdl * (float)il + w.dh * xdh * (float)ih;
    if (hh == 0) r -= w.ml * xsl + w.mh * xsh;
    return r;
}

// K-quant super-block `sb`, lane part j = lane & 7 (c = j/2, hh = j%2): its 16 qs bytes hold
// elements 64c+16hh+[0,16) (low nibbles, sub-block 2c) and 64c+32+16hh+[0,16) (high nibbles,
// sub-block 2c+1).  Activations from an ActRow (shared memory).
template <int FMT>
__device__ __forceinline__ float kq_part(uint4 hdr, uint4 qv, uint4 qh, int sb, int j,
                                         const ActRow &x) {
    const int c = j >> 1, hh = j & 1;
    const KqLane w = kq_unpack<FMT>(hdr, qv, qh, j);
    const int kl = sb * 256 + c * 64 + hh * 16;
    const int4 xa = *reinterpret_cast<const int4 *>(x.q + kl);
    const int4 xb = *reinterpret_cast<const int4 *>(x.q + kl + 32);
    const int bl = sb * 8 + 2 * c;
    return kq_dot(w, hh, xa, xb, x.d[bl], x.d[bl + 1], x.s[bl], x.s[bl + 1]);
}

// ------------------------------------------------------------------ Q6_K
//
// A Q6_K super-block (210 B) starts 2-byte aligned inside a 16-byte-aligned row.  Lane part j
// (c = j/2, hh = j%2; half h = c/2, c1 = c%2) covers, like the other K-quants, elements
// 64c+16hh+[0,16) and 64c+32+16hh+[0,16).  The first sixteen take their low bits from nibble c1
// of ql[64h+16hh+i], their high bits from bits 4c1, 4c1+1 of qh[32h+16hh+i] and scale
// sc[8h+4c1+hh]; the second sixteen nibble c1 of ql[64h+32+16hh+i], bits 4c1+2, 4c1+3 of the
// same qh bytes and scale sc[8h+4c1+2+hh].  The quants are kept as signed bytes q - 32, so the
// dot of a 16-weight piece is d*sc*xd*sum((q-32)*qx) with no offset term.

// 16 bytes at a 2-byte-aligned address (global or shared), as four little-endian words.
__device__ __forceinline__ uint4 ld16_a2(const uint8_t *p) {
    const uint16_t *h = reinterpret_cast<const uint16_t *>(p);
    return make_uint4((uint32_t)h[0] | ((uint32_t)h[1] << 16), (uint32_t)h[2] | ((uint32_t)h[3] << 16),
                      (uint32_t)h[4] | ((uint32_t)h[5] << 16), (uint32_t)h[6] | ((uint32_t)h[7] << 16));
}

// The quant words of one lane part: lo / hi = q - 32 of the two 16-weight pieces (signed bytes),
// and the two pieces' scales d*sc (exact in fp32: 11 x 8 bits).
struct Q6Lane {
    uint32_t lo[4], hi[4];
    float dl, dh;
};

__device__ __forceinline__ Q6Lane q6_unpack(const uint8_t *sbp, int j) {
    const int c = j >> 1, hh = j & 1, h = c >> 1, c1 = c & 1;
    const uint4 qa = ld16_a2(sbp + 64 * h + 16 * hh);
    const uint4 qb = ld16_a2(sbp + 64 * h + 32 + 16 * hh);
    const uint4 qh = ld16_a2(sbp + 128 + 32 * h + 16 * hh);
    const float d = half_bits_to_float(*reinterpret_cast<const uint16_t *>(sbp + 208));
    const int8_t *sc = reinterpret_cast<const int8_t *>(sbp + 192 + 8 * h + 4 * c1 + hh);
    Q6Lane r;
    r.dl = d * (float)sc[0];
    r.dh = d * (float)sc[2];
    const uint32_t a[4] = {qa.x, qa.y, qa.z, qa.w}, b[4] = {qb.x, qb.y, qb.z, qb.w};
    const uint32_t hb[4] = {qh.x, qh.y, qh.z, qh.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t lo6 = ((a[i] >> (4 * c1)) & 0x0F0F0F0Fu) | (((hb[i] >> (4 * c1)) & 0x03030303u) << 4);
        const uint32_t hi6 = ((b[i] >> (4 * c1)) & 0x0F0F0F0Fu) | (((hb[i] >> (4 * c1 + 2)) & 0x03030303u) << 4);
        r.lo[i] = __vsub4(lo6, 0x20202020u);
        r.hi[i] = __vsub4(hi6, 0x20202020u);
    }
    return r;
}

// The lane part's share of sum_k w_k * xhat_k (xa, xb: the activation bytes of the two pieces,
// xdl / xdh: the Q8_1 scales of their 32-blocks 2c and 2c+1).
__device__ __forceinline__ float q6_dot(const Q6Lane &w, int4 xa, int4 xb, float xdl, float xdh) {
    int il = __dp4a((int)w.lo[0], xa.x, 0);
    il = __dp4a((int)w.lo[1], xa.y, il);
    il = __dp4a((int)w.lo[2], xa.z, il);
    il = __dp4a((int)w.lo[3], xa.w, il);
    int ih = __dp4a((int)w.hi[0], xb.x, 0);
    ih = __dp4a((int)w.hi[1], xb.y, ih);
    ih = __dp4a((int)w.hi[2], xb.z, ih);
    ih = __dp4a((int)w.hi[3], xb.w, ih);
    return w.dl * xdl * (float)il + w.dh * xdh * (float)ih;
}

// Q8_0 block b of a row (34-byte blocks, 2-byte aligned): its 32 quants as 8 words and d.
struct Q80Block {
    uint32_t w[8];
    float d;
};

// Rows start 16-byte aligned, so block b starts on a word boundary when b is even and 2 bytes
// past one when b is odd: word loads cover it either way, none past the block's last byte.
__device__ __forceinline__ Q80Block q80_load(const uint8_t *row, int b) {
    const uint8_t *p = row + (size_t)b * kQ80Bytes;
    Q80Block r;
    if (b & 1) {   // p - 2 is aligned: d in the upper half of word 0, the quants in words 1..8
        const uint32_t w0 = ld_stream_u32(p - 2);
        r.d = half_bits_to_float(w0 >> 16);
#pragma unroll
        for (int i = 0; i < 8; i++) r.w[i] = ld_stream_u32(p + 2 + 4 * i);
    } else {       // p is aligned: d and the first 30 quants in 8 words, the last 2 quants alone
        uint32_t v[9];
#pragma unroll
        for (int i = 0; i < 8; i++) v[i] = ld_stream_u32(p + 4 * i);
        v[8] = ld_stream_u16(p + 32);
        r.d = half_bits_to_float(v[0]);
#pragma unroll
        for (int i = 0; i < 8; i++) r.w[i] = __funnelshift_r(v[i], v[i + 1], 16);
    }
    return r;
}

// sum over the block of (d*q) * (xd*qx); xq points at the block's 32 activation bytes.
__device__ __forceinline__ float q80_dot(const Q80Block &w, const int8_t *xq, float xd) {
    const int4 a = *reinterpret_cast<const int4 *>(xq);
    const int4 b = *reinterpret_cast<const int4 *>(xq + 16);
    int acc = __dp4a((int)w.w[0], a.x, 0);
    acc = __dp4a((int)w.w[1], a.y, acc);
    acc = __dp4a((int)w.w[2], a.z, acc);
    acc = __dp4a((int)w.w[3], a.w, acc);
    acc = __dp4a((int)w.w[4], b.x, acc);
    acc = __dp4a((int)w.w[5], b.y, acc);
    acc = __dp4a((int)w.w[6], b.z, acc);
    acc = __dp4a((int)w.w[7], b.w, acc);
    return w.d * xd * (float)acc;
}

// Q5_1 block b of a row (24-byte blocks; rows start 16-byte aligned, so every block is 8-byte
// aligned): its 32 five-bit quants as bytes (elements 4i..4i+3 in word i) and d, m.
struct Q51Block {
    uint32_t w[8];
    float d, m;
};

// Four consecutive bits of qh to bit 4 of four consecutive bytes.
__device__ __forceinline__ uint32_t q51_fifth(uint32_t qh, int n0) {
    return (((qh >> n0) & 0xFu) * 0x00204081u & 0x01010101u) << 4;
}

__device__ __forceinline__ Q51Block q51_unpack(uint2 h, uint2 a, uint2 c) {
    Q51Block r;
    r.d = half_bits_to_float(h.x & 0xFFFFu);
    r.m = half_bits_to_float(h.x >> 16);
    const uint32_t qh = h.y;
    const uint32_t qs[4] = {a.x, a.y, c.x, c.y};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        r.w[i] = (qs[i] & 0x0F0F0F0Fu) | q51_fifth(qh, 4 * i);
        r.w[4 + i] = ((qs[i] >> 4) & 0x0F0F0F0Fu) | q51_fifth(qh, 16 + 4 * i);
    }
    return r;
}

__device__ __forceinline__ Q51Block q51_load(const uint8_t *row, int b) {
    const uint8_t *p = row + (size_t)b * kQ51Bytes;
    return q51_unpack(ld_stream8(p), ld_stream8(p + 8), ld_stream8(p + 16));
}

// sum over the block of (d*q + m) * (xd*qx) = d*xd*sum(q*qx) + m*xs, xs = xd*sum(qx) exact.
__device__ __forceinline__ float q51_dot(const Q51Block &w, const int8_t *xq, float xd, float xs) {
    const int4 a = *reinterpret_cast<const int4 *>(xq);
    const int4 b = *reinterpret_cast<const int4 *>(xq + 16);
    int acc = __dp4a((int)w.w[0], a.x, 0);
    acc = __dp4a((int)w.w[1], a.y, acc);
    acc = __dp4a((int)w.w[2], a.z, acc);
    acc = __dp4a((int)w.w[3], a.w, acc);
    acc = __dp4a((int)w.w[4], b.x, acc);
    acc = __dp4a((int)w.w[5], b.y, acc);
    acc = __dp4a((int)w.w[6], b.z, acc);
    acc = __dp4a((int)w.w[7], b.w, acc);
    return fmaf(w.d * xd, (float)acc, w.m * xs);
}

// Whole-row partial dots for NT activation rows (lane's share; reduce across the warp after).
// x[t] for t < nt are valid; the rest are ignored.
template <int FMT, int NT>
__device__ __forceinline__ void row_parts(const uint8_t *row, int K, const ActRow *x, int nt,
                                          float *acc) {
    const int lane = threadIdx.x & 31;
    if (FMT == MOE_FMT_Q8_0) {
        for (int b = lane; b < K / 32; b += 32) {
            const Q80Block w = q80_load(row, b);
#pragma unroll
            for (int t = 0; t < NT; t++)
                if (t < nt) acc[t] += q80_dot(w, x[t].q + 32 * b, x[t].d[b]);
        }
        return;
    }
    if (FMT == MOE_FMT_Q5_1) {
        for (int b = lane; b < K / 32; b += 32) {
            const Q51Block w = q51_load(row, b);
#pragma unroll
            for (int t = 0; t < NT; t++)
                if (t < nt) acc[t] += q51_dot(w, x[t].q + 32 * b, x[t].d[b], x[t].s[b]);
        }
        return;
    }
    if (FMT == MOE_FMT_Q6_K) {
        const int j = lane & 7, c = j >> 1, hh = j & 1;
        for (int sb = lane >> 3; sb < K / 256; sb += 4) {
            const Q6Lane w = q6_unpack(row + (size_t)sb * kQ6KBytes, j);
            const int kl = sb * 256 + c * 64 + hh * 16, bl = sb * 8 + 2 * c;
#pragma unroll
            for (int t = 0; t < NT; t++)
                if (t < nt)
                    acc[t] += q6_dot(w, *reinterpret_cast<const int4 *>(x[t].q + kl),
                                     *reinterpret_cast<const int4 *>(x[t].q + kl + 32),
                                     x[t].d[bl], x[t].d[bl + 1]);
        }
        return;
    }
    constexpr int SBB = FMT == MOE_FMT_Q5_K ? kQ5KBytes : kQ4KBytes;
    constexpr int QS = FMT == MOE_FMT_Q5_K ? 48 : 16;
    const int nsb = K / 256;
    const int j = lane & 7;
    // up to 4 groups of 4 super-blocks (K <= 4096): issue every load before the math
    uint4 hdr[4], qv[4], qh[4];
#pragma unroll
    for (int g = 0; g < 4; g++) {
        const int sb = g * 4 + (lane >> 3);
        hdr[g] = make_uint4(0, 0, 0, 0);
        qv[g] = hdr[g];
        qh[g] = hdr[g];
        if (sb < nsb) {
            const uint8_t *p = row + (size_t)sb * SBB;
            hdr[g] = ld_stream16(p);
            qv[g] = ld_stream16(p + QS + 16 * j);
            if (FMT == MOE_FMT_Q5_K) qh[g] = ld_stream16(p + 16 + 16 * (j & 1));
        }
    }
#pragma unroll
    for (int g = 0; g < 4; g++) {
        const int sb = g * 4 + (lane >> 3);
        if (sb < nsb) {
#pragma unroll
            for (int t = 0; t < NT; t++)
                if (t < nt) acc[t] += kq_part<FMT>(hdr[g], qv[g], qh[g], sb, j, x[t]);
        }
    }
}

template <int NT>
__device__ __forceinline__ void row_parts_fmt(int fmt, const uint8_t *row, int K, const ActRow *x,
                                              int nt, float *acc) {
    if (fmt == MOE_FMT_Q4_K) row_parts<MOE_FMT_Q4_K, NT>(row, K, x, nt, acc);
    else if (fmt == MOE_FMT_Q5_K) row_parts<MOE_FMT_Q5_K, NT>(row, K, x, nt, acc);
    else if (fmt == MOE_FMT_Q8_0) row_parts<MOE_FMT_Q8_0, NT>(row, K, x, nt, acc);
    else if (fmt == MOE_FMT_Q6_K) row_parts<MOE_FMT_Q6_K, NT>(row, K, x, nt, acc);
    else row_parts<MOE_FMT_Q5_1, NT>(row, K, x, nt, acc);
}

// Q8_1 of 32 values, one per lane (the h of one 32-row block of one slot).
__device__ __forceinline__ void q8_1_warp32(float v, int8_t *q, uint16_t *d16, uint16_t *s16,
                                            float *dsum, uint32_t *status) {
    const int lane = threadIdx.x & 31;
    bool fin = isfinite(v);
    float a = fabsf(v);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(kFullMask, a, o));
    fin = __all_sync(kFullMask, fin);
    const float d = __fdiv_rn(a, 127.0f);
    int qi = 0;
    if (fin && d != 0.0f) qi = max(-127, min(127, (int)roundf(__fdiv_rn(v, d))));
    int sum = qi;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(kFullMask, sum, o);
    q[lane] = (int8_t)qi;
    if (lane == 0) {
        if (fin) {
            const __half dh = __float2half_rn(d);
            *d16 = __half_as_ushort(dh);
            *s16 = __half_as_ushort(__float2half_rn(__fmul_rn(d, (float)sum)));
            *dsum = __fmul_rn(__half2float(dh), (float)sum);
        } else {
            *d16 = 0;
            *s16 = 0;
            *dsum = 0.0f;
            set_status(status, MOE_ERR_NONFINITE);
        }
    }
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

}  // namespace moe
