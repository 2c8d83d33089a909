/*
 * moe_oracle.c -- plain, slow, obviously correct CPU oracle of the quantized MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's CPU-baseline leg
 * are the only callers.  The product (the CUDA library) never links, loads or calls this file,
 * and this file includes no header of the product: every constant and layout below is written
 * out here a second time from the block-format definitions, on purpose.
 *
 * What it computes (the layer of "Strata: a 125B MoE at 94 tok/s on a 12 GB Card", section
 * "Three architecture facts": experts per layer, routed + shared; the per-expert formats of the
 * "Strata v0.1.31" release notes, section "Experimental: Unsloth UD-Q4_K_XL on a normal PC":
 * Q4_K, Q5_K, Q5_1 and Q8_0 experts whose dequantizers follow llama.cpp's bit for bit; the q8_1
 * activations of the "Strata v0.1.39" release notes, fixes list, #606):
 *
 *   O1  block decode (Q4_K, Q5_K, Q5_1, Q8_0, Q6_K) to exact fp64 and to the fp32 value
 *       RN32( RN32(d*sc)*q - RN32(dmin*m) )             (Q8_0: RN32(d*q); Q5_1: RN32(d*q + m);
 *       Q6_K: RN32(RN32(d*sc)*q) -- the format real Q4_K_M model files mix in)
 *   O2  Q8_1 quantization of 32-value blocks: amax, d = amax/127 (fp32 division),
 *       q = round-half-away(x/d) clamped to [-127,127], stored d16 = fp16(d),
 *       s16 = fp16(d * sum(q)); a block holding a non-finite value becomes all zero
 *   O3  top-k of the router logits (descending logit, ties to the lower expert id) and the
 *       softmax over the chosen k logits, in fp64, stored as fp32
 *   O4  histogram of the chosen experts, exclusive prefix sum, stable permutation
 *   O5  gate/up rows times the dequantized Q8_1 activations, in fp64, from the exact weights
 *   O6  SwiGLU: h = g / (1 + exp(-g)) * u, in fp64
 *   O7  Q8_1 of fp32(h), zero-padded to the down rows' stored width
 *   O8  down rows times the dequantized Q8_1(h), in fp64
 *   O9  out[t] = sum_j w[t][j] * y[t][e_j] + y[t][shared], in fp64, stored as fp32
 *   O10 router logits[t][e] = sum_h x[t][h] * Wr[e][h] of the fp32 hidden state and fp32
 *       router rows, summed in fp64 in h order, stored as fp32 (the per-token router the
 *       engine keeps on the GPU, "Strata: a 125B MoE at 94 tok/s on a 12 GB Card")
 *   O11 optional shared-expert gate: g[t] = 1 / (1 + exp(-sum_h x[t][h] * wg[h])) in fp64;
 *       with it, O9's shared term is g[t] * y[t][shared]
 *
 * Nothing here is blocked, fused or reordered beyond these definitions.  The rows of one expert
 * matrix may be computed on several OpenMP threads; every sum runs in the same order whatever
 * the thread count.
 *
 * Pinned by tests/test_oracle_pins.py (hand-computed blocks, a 64x64 scale pack/unpack round
 * trip, exact-rational rounding, Q8_1 closed forms, brute-force top-k, grouping invariants and
 * dense-fp64 numpy FFNs on tiny layers).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_Q4_K = 0, ORC_Q5_K = 1, ORC_Q8_0 = 2, ORC_Q5_1 = 3, ORC_Q6_K = 4 };

/* weights and bytes per block of each format */
static int orc_block_weights(int fmt) { return fmt == ORC_Q8_0 || fmt == ORC_Q5_1 ? 32 : 256; }
static int orc_block_bytes(int fmt) {
    return fmt == ORC_Q4_K ? 144 : fmt == ORC_Q5_K ? 176 : fmt == ORC_Q8_0 ? 34 : fmt == ORC_Q5_1 ? 24 : 210;
}

int oracle_block_weights(int fmt) { return fmt >= 0 && fmt <= 4 ? orc_block_weights(fmt) : -1; }
int oracle_block_bytes(int fmt) { return fmt >= 0 && fmt <= 4 ? orc_block_bytes(fmt) : -1; }

/* ---------------------------------------------------------------- IEEE binary16 <-> binary64 */

/* Exact value of a binary16 bit pattern. */
static double orc_half_to_double(uint16_t h) {
    int sign = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m | 1024), e - 25);     /* (1024 + m) * 2^(e - 15 - 10) */
    return sign ? -v : v;
}

/* binary32 -> binary16, round to nearest, ties to even. */
static uint16_t orc_float_to_half(float f) {
    double v = fabs((double)f);
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    if (isnan(f)) return sign | 0x7e00;
    if (isinf(f)) return sign | 0x7c00;
    if (v < ldexp(1.0, -14)) {                     /* subnormal range: multiples of 2^-24 */
        double r = nearbyint(ldexp(v, 24));        /* default mode: nearest, ties to even */
        return sign | (uint16_t)r;                 /* r == 1024 is the smallest normal */
    }
    int ex;
    frexp(v, &ex);                                 /* v in [2^(ex-1), 2^ex) */
    int E = ex - 1;
    double s = nearbyint(ldexp(v, 10 - E));        /* significand scaled to [1024, 2048] */
    if (s == 2048.0) { s = 1024.0; E += 1; }
    if (E > 15) return sign | 0x7c00;              /* overflow to infinity */
    return sign | (uint16_t)(((E + 15) << 10) | ((int)s - 1024));
}

double oracle_half_to_double(uint16_t h) { return orc_half_to_double(h); }
uint16_t oracle_float_to_half(float f) { return orc_float_to_half(f); }

/* ------------------------------------------------------------------------ O1: block decode */

/* 6-bit scale and min of sub-block j (0..7) from the 12 packed bytes S of a K-quant block:
 * j < 4 : sc = S[j] & 63,                        m = S[j+4] & 63
 * j >= 4: sc = (S[j+4] & 15) | ((S[j-4] >> 6) << 4),
 *         m  = (S[j+4] >> 4) | ((S[j]   >> 6) << 4)                                          */
static void orc_kquant_scale_min(const uint8_t *S, int j, int *sc, int *m) {
    if (j < 4) {
        *sc = S[j] & 63;
        *m = S[j + 4] & 63;
    } else {
        *sc = (S[j + 4] & 15) | ((S[j - 4] >> 6) << 4);
        *m = (S[j + 4] >> 4) | ((S[j] >> 6) << 4);
    }
}

/* Decode one block into w64[0..bw) (exact) and w32[0..bw) (fp32 as defined in O1).
 * Q4_K (144 B): d, dmin (fp16, bytes 0-3), S[12] (4-15), qs[128] (16-143).
 *   element n: c = n / 64, r = n % 64; r < 32 -> sub-block 2c, q = low nibble of qs[32c + r];
 *   r >= 32 -> sub-block 2c+1, q = high nibble of qs[32c + r - 32].
 * Q5_K (176 B): d, dmin, S as Q4_K; qh[32] (16-47); qs[128] (48-175); the fifth bit of
 *   element n is bit (2c) of qh[r] for r < 32 and bit (2c+1) of qh[r-32] for r >= 32.
 * Q8_0 (34 B): d (fp16), q[32] int8.
 * Q5_1 (24 B): d, m (fp16, bytes 0-3), qh (32 bits, little endian, bytes 4-7), qs[16] (8-23);
 *   element n < 16: q = low nibble of qs[n], n >= 16: high nibble of qs[n-16]; bit n of qh is
 *   the fifth bit of element n; w = d*q + m (d*q has <= 16 significant bits, so the fp32 value
 *   is RN32(d*q + m) whether or not the multiply-add is fused).
 * Q6_K (210 B): ql[128] (bytes 0-127, low 4 bits), qh[64] (128-191, high 2 bits), sc[16]
 *   (192-207, int8, one per 16 weights), d (fp16, 208-209).  Element n: half h = n / 128,
 *   i = n % 128, quarter g = i / 32, l = i % 32; low bits = nibble of ql[64h + l + 32(g & 1)]
 *   (low nibble for g < 2, high for g >= 2); high bits = bits 2g, 2g+1 of qh[32h + l];
 *   q = low + 16 high - 32; scale sc[8h + 2g + l / 16]; w = RN32( RN32(d*sc) * q ), where
 *   d*sc is exact (11 x 8 bits) and the product with q rounds once.                           */
static void orc_decode_block(int fmt, const uint8_t *b, double *w64, float *w32) {
    if (fmt == ORC_Q6_K) {
        double d = orc_half_to_double((uint16_t)(b[208] | (b[209] << 8)));
        for (int n = 0; n < 256; n++) {
            int h = n / 128, i = n % 128, g = i / 32, l = i % 32;
            int lo = b[64 * h + l + 32 * (g & 1)];
            lo = g < 2 ? (lo & 15) : (lo >> 4);
            int hi = (b[128 + 32 * h + l] >> (2 * g)) & 3;
            int q = lo + 16 * hi - 32;
            int sc = (int8_t)b[192 + 8 * h + 2 * g + l / 16];
            float d1 = (float)(d * sc);             /* exact */
            w64[n] = (double)d1 * q;
            if (w32) w32[n] = d1 * (float)q;
        }
        return;
    }
    if (fmt == ORC_Q5_1) {
        double d = orc_half_to_double((uint16_t)(b[0] | (b[1] << 8)));
        double m = orc_half_to_double((uint16_t)(b[2] | (b[3] << 8)));
        uint32_t qh = (uint32_t)b[4] | ((uint32_t)b[5] << 8) | ((uint32_t)b[6] << 16) |
                      ((uint32_t)b[7] << 24);
        for (int n = 0; n < 32; n++) {
            int q = n < 16 ? (b[8 + n] & 15) : (b[8 + n - 16] >> 4);
            q |= (int)((qh >> n) & 1u) << 4;
            w64[n] = d * q + m;
            if (w32) w32[n] = fmaf((float)d, (float)q, (float)m);
        }
        return;
    }
    if (fmt == ORC_Q8_0) {
        double d = orc_half_to_double((uint16_t)(b[0] | (b[1] << 8)));
        for (int n = 0; n < 32; n++) {
            int q = (int8_t)b[2 + n];
            w64[n] = d * q;
            if (w32) w32[n] = (float)(d * q);        /* exact: 11 x 8 significant bits */
        }
        return;
    }
    double d = orc_half_to_double((uint16_t)(b[0] | (b[1] << 8)));
    double dmin = orc_half_to_double((uint16_t)(b[2] | (b[3] << 8)));
    const uint8_t *S = b + 4;
    const uint8_t *qh = fmt == ORC_Q5_K ? b + 16 : NULL;
    const uint8_t *qs = fmt == ORC_Q5_K ? b + 48 : b + 16;
    for (int n = 0; n < 256; n++) {
        int c = n / 64, r = n % 64, j, q;
        if (r < 32) {
            j = 2 * c;
            q = qs[32 * c + r] & 15;
            if (qh) q += 16 * ((qh[r] >> (2 * c)) & 1);
        } else {
            j = 2 * c + 1;
            q = qs[32 * c + r - 32] >> 4;
            if (qh) q += 16 * ((qh[r - 32] >> (2 * c + 1)) & 1);
        }
        int sc, m;
        orc_kquant_scale_min(S, j, &sc, &m);
        float d1 = (float)(d * sc);                 /* exact: 11 x 6 significant bits */
        float m1 = (float)(dmin * m);               /* exact */
        w64[n] = (double)d1 * q - (double)m1;
        if (w32) w32[n] = fmaf(d1, (float)q, -m1);  /* one rounding of d1*q - m1 */
    }
}

/* O1 over a packed row of nblocks blocks.  Returns 0, or -1 for an unknown format. */
int oracle_dequant_row(int fmt, const uint8_t *row, int64_t nblocks, double *w64, float *w32) {
    if (fmt < 0 || fmt > 4) return -1;
    int bw = orc_block_weights(fmt), bb = orc_block_bytes(fmt);
    for (int64_t i = 0; i < nblocks; i++)
        orc_decode_block(fmt, row + i * bb, w64 + i * bw, w32 ? w32 + i * bw : NULL);
    return 0;
}

/* ------------------------------------------------------------------------ O2: Q8_1 blocks */

/* Quantize nblocks blocks of 32 fp32 values.  Returns the number of blocks that held a
 * non-finite value (each written as q = 0, d = s = 0).                                        */
int64_t oracle_quantize_q8_1(const float *x, int64_t nblocks, int8_t *q, uint16_t *d16,
                             uint16_t *s16) {
    int64_t bad = 0;
    for (int64_t b = 0; b < nblocks; b++) {
        const float *xb = x + 32 * b;
        int8_t *qb = q + 32 * b;
        int finite = 1;
        float amax = 0.0f;
        for (int i = 0; i < 32; i++) {
            if (!isfinite(xb[i])) finite = 0;
            else if (fabsf(xb[i]) > amax) amax = fabsf(xb[i]);
        }
        if (!finite) {
            memset(qb, 0, 32);
            d16[b] = 0;
            s16[b] = 0;
            bad++;
            continue;
        }
        float d = amax / 127.0f;                    /* one IEEE fp32 division */
        int sum = 0;
        for (int i = 0; i < 32; i++) {
            int qi = 0;
            if (d != 0.0f) {
                float r = xb[i] / d;                /* one IEEE fp32 division */
                qi = (int)roundf(r);                /* half away from zero */
                if (qi > 127) qi = 127;
                if (qi < -127) qi = -127;
            }
            qb[i] = (int8_t)qi;
            sum += qi;
        }
        d16[b] = orc_float_to_half(d);
        s16[b] = orc_float_to_half(d * (float)sum); /* sum is exact in fp32 */
    }
    return bad;
}

/* ------------------------------------------------------------------------ O3: router top-k */

/* For each of T tokens choose k of E experts: descending logit, ties to the lower id.  The
 * weights are the softmax over the chosen logits, in fp64, stored as fp32.  Returns the number
 * of tokens whose logits held a non-finite value (their ids are 0..k-1, weights 1/k).        */
int oracle_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w) {
    int bad = 0;
    char *taken = (char *)malloc((size_t)E);
    for (int t = 0; t < T; t++) {
        const float *l = logits + (int64_t)t * E;
        int finite = 1;
        for (int e = 0; e < E; e++)
            if (!isfinite(l[e])) finite = 0;
        if (!finite) {
            for (int j = 0; j < k; j++) {
                ids[(int64_t)t * k + j] = j;
                w[(int64_t)t * k + j] = 1.0f / (float)k;
            }
            bad++;
            continue;
        }
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; j++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict '>' keeps the lower id */
            }
            taken[best] = 1;
            ids[(int64_t)t * k + j] = best;
        }
        double lmax = l[ids[(int64_t)t * k]];
        double den = 0.0;
        for (int j = 0; j < k; j++) den += exp((double)l[ids[(int64_t)t * k + j]] - lmax);
        for (int j = 0; j < k; j++)
            w[(int64_t)t * k + j] = (float)(exp((double)l[ids[(int64_t)t * k + j]] - lmax) / den);
    }
    free(taken);
    return bad;
}

/* ------------------------------------------------------------------------ O4: grouping */

/* counts[e] = #{(t,j): ids[t][j] = e}; offsets = exclusive prefix sum (E+1 entries);
 * perm[offsets[e] + r] = t*k + j for the r-th such pair in ascending t (then j);
 * inv_perm[perm[i]] = i.  Returns -1 if an id is out of range.                                */
int oracle_group(const int32_t *ids, int T, int k, int E, int32_t *counts, int32_t *offsets,
                 int32_t *perm, int32_t *inv_perm) {
    int64_t A = (int64_t)T * k;
    if (E <= 0 || T < 0 || k < 0) return -1;
    for (int e = 0; e < E; e++) counts[e] = 0;
    for (int64_t a = 0; a < A; a++) {
        if (ids[a] < 0 || ids[a] >= E) return -1;
        counts[ids[a]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    if (!fill) return -1;
    for (int64_t a = 0; a < A; a++) {               /* ascending a = ascending t, then j */
        int e = ids[a];
        int64_t i = offsets[e] + fill[e]++;
        perm[i] = (int32_t)a;
        inv_perm[a] = (int32_t)i;
    }
    free(fill);
    return 0;
}

/* ------------------------------------------------------------------------ O5-O9: the FFN */

/* One expert's three matrices inside a host arena.  fmt: 0 Q4_K, 1 Q5_K, 2 Q8_0, 3 Q5_1, 4 Q6_K.
 * gate, up: ffn rows of hidden weights; down: hidden rows of ffn weights (padded to whole
 * blocks).  Offsets and row strides are in bytes.                                             */
typedef struct {
    int32_t fmt;
    int32_t reserved;
    int64_t off[3];    /* gate, up, down */
    int64_t stride[3];
} oracle_expert;

/* Dense fp64 dot of one packed row (nblocks blocks) with a vector. */
static double orc_row_dot(int fmt, const uint8_t *row, int64_t nblocks, const double *v,
                          double *scratch) {
    oracle_dequant_row(fmt, row, nblocks, scratch, NULL);
    int64_t n = nblocks * orc_block_weights(fmt);
    double acc = 0.0;
    for (int64_t i = 0; i < n; i++) acc += scratch[i] * v[i];
    return acc;
}

/* Dequantized Q8_1 vector: xhat[i] = fp16->fp64(d16[i/32]) * q[i]. */
static void orc_q8_1_values(const int8_t *q, const uint16_t *d16, int64_t n, double *xhat) {
    for (int64_t i = 0; i < n; i++) xhat[i] = orc_half_to_double(d16[i / 32]) * q[i];
}

/* Stored width (in weights) of a down row of `ffn` weights: whole blocks. */
static int64_t orc_padded(int fmt, int64_t ffn) {
    int64_t bw = orc_block_weights(fmt);
    return (ffn + bw - 1) / bw * bw;
}

/* O5-O8 for one token and one expert.  xhat: the token's dequantized Q8_1 activations
 * [hidden].  Writes g, u, h [ffn] (fp64), the Q8_1 of fp32(h) padded to the down width
 * (hq [fp], hd/hs [fp/32]) and y [hidden] (fp64).  Any output pointer may be NULL except y.  */
int oracle_expert_ffn(const uint8_t *arena, const oracle_expert *ex, int hidden, int ffn,
                      const double *xhat, double *g, double *u, double *h, int8_t *hq,
                      uint16_t *hd, uint16_t *hs, double *y) {
    int fmt = ex->fmt;
    if (fmt < 0 || fmt > 4) return -1;
    int bw = orc_block_weights(fmt);
    if (hidden % bw) return -1;
    int64_t fp = orc_padded(fmt, ffn);
    int64_t nb_in = hidden / bw, nb_down = fp / bw;
    double *hh = (double *)calloc((size_t)ffn, sizeof(double));
    float *hf = (float *)calloc((size_t)fp, sizeof(float));
    int8_t *q = (int8_t *)malloc((size_t)fp);
    uint16_t *dd = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(fp / 32));
    uint16_t *ss = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(fp / 32));
    double *hhat = (double *)malloc(sizeof(double) * (size_t)fp);

    /* rows are independent: the row loops may run on several threads (each row's sum is the
     * same sequential loop whatever the thread count) */
#pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)(hidden > fp ? hidden : fp));
#pragma omp for schedule(static)
        for (int r = 0; r < ffn; r++) {
            double gr = orc_row_dot(fmt, arena + ex->off[0] + r * ex->stride[0], nb_in, xhat, sc);
            double ur = orc_row_dot(fmt, arena + ex->off[1] + r * ex->stride[1], nb_in, xhat, sc);
            double hr = gr / (1.0 + exp(-gr)) * ur;                 /* O6 */
            if (g) g[r] = gr;
            if (u) u[r] = ur;
            hh[r] = hr;
            hf[r] = (float)hr;
        }
        free(sc);
    }
    if (h) memcpy(h, hh, sizeof(double) * (size_t)ffn);
    oracle_quantize_q8_1(hf, fp / 32, q, dd, ss);                   /* O7 (tail stays zero) */
    orc_q8_1_values(q, dd, fp, hhat);
    if (hq) memcpy(hq, q, (size_t)fp);
    if (hd) memcpy(hd, dd, sizeof(uint16_t) * (size_t)(fp / 32));
    if (hs) memcpy(hs, ss, sizeof(uint16_t) * (size_t)(fp / 32));
#pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)(hidden > fp ? hidden : fp));
#pragma omp for schedule(static)
        for (int i = 0; i < hidden; i++)                             /* O8 */
            y[i] = orc_row_dot(fmt, arena + ex->off[2] + i * ex->stride[2], nb_down, hhat, sc);
        free(sc);
    }

    free(hh); free(hf); free(q); free(dd); free(ss); free(hhat);
    return 0;
}

/* O8-O9 from Q8_1(h) rows given from outside (the reading that checks a layer whose h was
 * computed elsewhere in two parts: h itself, and everything after it).  Slot s belongs to token
 * slot_tok[s] and expert slot_exp[s] with routing weight slot_w[s]; its h^ is the dequantized
 * Q8_1 row hq [s][0..fp), hd [s][0..fp/32) (fp = the expert's stored down width, <= hpad).
 * y = W_down h^ (exact weights, fp64) and out64[tok] += w * y, slot after slot in the order
 * given.  out64 [T][hidden] is overwritten.  Returns 0, or -1 for bad arguments.             */
int oracle_down_combine(const uint8_t *arena, const oracle_expert *experts, int n_experts,
                        int hidden, int ffn, const int8_t *hq, const uint16_t *hd, int hpad,
                        const int32_t *slot_tok, const int32_t *slot_exp, const double *slot_w,
                        int n_slots, int T, double *out64) {
    if (!arena || !experts || !hq || !hd || !slot_tok || !slot_exp || !slot_w || !out64) return -1;
    if (hidden <= 0 || ffn <= 0 || hpad % 32 || n_slots < 0 || T <= 0) return -1;
    memset(out64, 0, sizeof(double) * (size_t)T * (size_t)hidden);
    double *hhat = (double *)malloc(sizeof(double) * (size_t)hpad);
    double *y = (double *)malloc(sizeof(double) * (size_t)hidden);
    int err = 0;
    for (int s = 0; s < n_slots && !err; s++) {
        const int t = slot_tok[s], e = slot_exp[s];
        if (t < 0 || t >= T || e < 0 || e >= n_experts) { err = -1; break; }
        const oracle_expert *ex = &experts[e];
        const int64_t fp = orc_padded(ex->fmt, ffn);
        if (fp > hpad) { err = -1; break; }
        orc_q8_1_values(hq + (int64_t)s * hpad, hd + (int64_t)s * (hpad / 32), fp, hhat);
        const int64_t nb_down = fp / orc_block_weights(ex->fmt);
#pragma omp parallel
        {
            double *sc = (double *)malloc(sizeof(double) * (size_t)fp);
#pragma omp for schedule(static)
            for (int i = 0; i < hidden; i++)                                     /* O8 */
                y[i] = orc_row_dot(ex->fmt, arena + ex->off[2] + i * ex->stride[2], nb_down, hhat,
                                   sc);
            free(sc);
        }
        for (int i = 0; i < hidden; i++) out64[(int64_t)t * hidden + i] += slot_w[s] * y[i];   /* O9 */
    }
    free(hhat);
    free(y);
    return err;
}

/* O10: logits [T][E] (fp32, and the fp64 sums when l64 is not NULL) of x [T][H] and the
 * router rows Wr [E][H].  Returns 0, or -1 for bad arguments.                                */
int oracle_router(const float *x, const float *Wr, int T, int H, int E, float *l32,
                  double *l64) {
    if (T < 0 || H <= 0 || E <= 0 || !x || !Wr || !l32) return -1;
    for (int t = 0; t < T; t++) {
        for (int e = 0; e < E; e++) {
            double s = 0.0;
            for (int h = 0; h < H; h++)
                s += (double)x[(int64_t)t * H + h] * (double)Wr[(int64_t)e * H + h];
            l32[(int64_t)t * E + e] = (float)s;
            if (l64) l64[(int64_t)t * E + e] = s;
        }
    }
    return 0;
}

/* O11: the shared-expert gate g [T] of x [T][H] and the gate row wg [H], in fp64.           */
int oracle_shared_gate(const float *x, const float *wg, int T, int H, double *g) {
    if (T < 0 || H <= 0 || !x || !wg || !g) return -1;
    for (int t = 0; t < T; t++) {
        double s = 0.0;
        for (int h = 0; h < H; h++) s += (double)x[(int64_t)t * H + h] * (double)wg[h];
        g[t] = 1.0 / (1.0 + exp(-s));
    }
    return 0;
}

static int orc_forward(const uint8_t *arena, const oracle_expert *experts, int n_experts,
                       int shared, int hidden, int ffn, const float *x, const int32_t *ids,
                       const float *w, int T, int k, const int32_t *tokens, int n_tokens,
                       const double *gate, float *out, double *out64);

/* O1-O9 for a list of tokens.  x [T][hidden], ids/w [T][k] (from O3); experts[0..E) routed,
 * experts[shared] the always-on shared expert (shared < 0: none).  tokens[0..n_tokens) names
 * the tokens to compute (NULL: all T in order); out/out64 get one row [hidden] per listed
 * token.  Returns 0, or -1 for bad arguments.                                                 */
int oracle_forward(const uint8_t *arena, const oracle_expert *experts, int n_experts, int shared,
                   int hidden, int ffn, const float *x, const int32_t *ids, const float *w, int T,
                   int k, const int32_t *tokens, int n_tokens, float *out, double *out64) {
    return orc_forward(arena, experts, n_experts, shared, hidden, ffn, x, ids, w, T, k, tokens,
                       n_tokens, NULL, out, out64);
}

/* The same with the O11 gate on the shared expert: gate [T] (from oracle_shared_gate).       */
int oracle_forward_gated(const uint8_t *arena, const oracle_expert *experts, int n_experts,
                         int shared, int hidden, int ffn, const float *x, const int32_t *ids,
                         const float *w, int T, int k, const int32_t *tokens, int n_tokens,
                         const double *gate, float *out, double *out64) {
    if (!gate) return -1;
    return orc_forward(arena, experts, n_experts, shared, hidden, ffn, x, ids, w, T, k, tokens,
                       n_tokens, gate, out, out64);
}

static int orc_forward(const uint8_t *arena, const oracle_expert *experts, int n_experts,
                       int shared, int hidden, int ffn, const float *x, const int32_t *ids,
                       const float *w, int T, int k, const int32_t *tokens, int n_tokens,
                       const double *gate, float *out, double *out64) {
    if (hidden % 32 || n_tokens < 0) return -1;
    if (!tokens) n_tokens = T;
    int err = 0;
    /* tokens in order; the threads work inside each expert's row loops (oracle_expert_ffn) */
    for (int it = 0; it < n_tokens; it++) {
        int t = tokens ? tokens[it] : it;
        if (t < 0 || t >= T) { err = -1; continue; }
        int8_t *q = (int8_t *)malloc((size_t)hidden);
        uint16_t *d16 = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(hidden / 32));
        uint16_t *s16 = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(hidden / 32));
        double *xhat = (double *)malloc(sizeof(double) * (size_t)hidden);
        double *y = (double *)malloc(sizeof(double) * (size_t)hidden);
        double *acc = (double *)calloc((size_t)hidden, sizeof(double));
        oracle_quantize_q8_1(x + (int64_t)t * hidden, hidden / 32, q, d16, s16);   /* O2 */
        orc_q8_1_values(q, d16, hidden, xhat);
        for (int j = 0; j <= k; j++) {
            int e;
            double wt;
            if (j < k) {
                e = ids[(int64_t)t * k + j];
                wt = (double)w[(int64_t)t * k + j];
            } else {
                if (shared < 0) break;
                e = shared;
                wt = gate ? gate[t] : 1.0;                               /* O11 or no gate */
            }
            if (e < 0 || e >= n_experts || oracle_expert_ffn(arena, &experts[e], hidden, ffn,
                                                             xhat, NULL, NULL, NULL, NULL,
                                                             NULL, NULL, y)) {
                err = -1;
                break;
            }
            for (int i = 0; i < hidden; i++) acc[i] += wt * y[i];       /* O9 */
        }
        for (int i = 0; i < hidden; i++) {
            if (out) out[(int64_t)it * hidden + i] = (float)acc[i];
            if (out64) out64[(int64_t)it * hidden + i] = acc[i];
        }
        free(q); free(d16); free(s16); free(xhat); free(y); free(acc);
    }
    return err;
}

/* Thread control for the CPU-baseline timing (0: leave the OpenMP default). */
int oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
