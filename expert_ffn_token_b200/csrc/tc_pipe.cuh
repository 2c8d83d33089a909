// tc_pipe.cuh -- pieces shared by the two tensor-core projection kernels (k_gateup_tc.cu,
// k_down_tc.cu): the arguments, the job-major tile walk, mbarrier rings with bounded waits, and
// the fp16-pair and quantizer helpers.
#pragma once

#include <cuda.h>

#include "moe_internal.cuh"
#include "tc.cuh"

namespace moe {
namespace tcp {

using namespace ptx;

// Bytes of 256 packed weights of each format (Q8_0: eight 34-byte blocks, Q5_1: eight 24-byte).
__host__ __device__ inline uint32_t sb_bytes(int fmt) {
    return fmt == MOE_FMT_Q4_K ? 144u : fmt == MOE_FMT_Q5_K ? 176u : fmt == MOE_FMT_Q8_0 ? 272u : 192u;
}
__host__ __device__ inline bool has_min(int fmt) { return fmt != MOE_FMT_Q8_0; }

struct GemmArgs {
    const CUtensorMap *wmaps;     // [n_experts (+ shared)][3]: packed gate, up, down
    const ExpertDev *experts;
    const Job *jobs;
    const int32_t *njobs;
    const int32_t *perm;
    const float *w;
    const __half *act;            // gate/up: x^ hi [T][H]; down: h^ [slots][Kd] (fp16 rows)
    const __half *act_lo;         // gate/up: x^ lo [T][H] (x^ = hi + lo exactly)
    const float *xs_hi, *xs_lo;   // gate/up: block sums xd * sum(q) [T][H/32], tf32 hi + lo
    const float *act_scale;       // 2^e per row of act
    const int8_t *xq;             // gate/up, kind::i8: Q8_1 quants of x [T][H]
    const uint16_t *xd;           //   their fp16 block scales [T][H/32]
    const float *xsum;            //   block sums xd * sum(q) [T][H/32]
    int act_pitch;                // elements per row of act
    int T, k, H, F, hpad;
    int nst;                      // 64-wide contraction stages per tile
    int mt_count;                 // weight-row tiles per token slice
    int tn;                       // tokens per tile
    int DA, DB, DR, lag;          // ring depths and activation stages in flight
    int DK, DC;                   // kind::i8 gate/up: row-constant and column-constant rings
    uint32_t rawb;                // bytes of one packed stage (128 rows x largest super-block)
    // gate/up outputs: Q8_1(h) per slot, optional fp32 h
    int8_t *hq;
    uint16_t *hd, *hs;
    float *hsum;
    float *h;
    // down outputs
    float *out;
    const float *gate;            // optional [T]: the shared expert's weight per token
    float *y;                     // deterministic mode: y per slot
    uint32_t *status;
    uint64_t wait_ns;
};

// A ring position: slot s of depth d, phase parity ph.
struct Ring {
    int s = 0;
    uint32_t ph = 0;
    __device__ __forceinline__ void adv(int n, int d) {
        s += n;
        while (s >= d) {
            s -= d;
            ph ^= 1u;
        }
    }
};

struct Tile {
    int e, fmt, mt, slot_base, n_valid, n_mma, shared;
};

struct Cursor {
    int j = 0, base = 0;
};

// Tile i of the job-major order (job, token slice of a.tn, weight-row tile), i increasing.
__device__ __forceinline__ bool tile_at(const GemmArgs &a, int nj, Cursor &c, int i, Tile &t) {
    while (c.j < nj) {
        const Job jb = a.jobs[c.j];
        const int ns = (jb.n + a.tn - 1) / a.tn;
        const int cnt = ns * a.mt_count;
        if (i < c.base + cnt) {
            const int rel = i - c.base;
            const int sl = rel / a.mt_count;
            t.mt = rel - sl * a.mt_count;
            t.e = jb.expert;
            t.fmt = a.experts[jb.expert].fmt;
            t.slot_base = jb.slot0 + sl * a.tn;
            t.n_valid = min(a.tn, jb.n - sl * a.tn);
            t.n_mma = (t.n_valid + 15) & ~15;
            t.shared = jb.shared;
            return true;
        }
        c.base += cnt;
        c.j++;
    }
    return false;
}

// Bounded wait on phase `parity` of `bar`; false once this CTA is aborting.  A wait that runs
// out sets the CTA's abort flag and MOE_ERR_TIMEOUT.
static __device__ __noinline__ bool wait_slow(uint64_t *bar, uint32_t parity, int *abort,
                                              uint32_t *status, uint64_t limit) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (*(volatile int *)abort) return false;
        if (globaltimer() - t0 > limit) {
            *(volatile int *)abort = 1;
            set_status(status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ bool wait1(const GemmArgs &a, int *abort, uint64_t *bar,
                                      uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_slow(bar, parity, abort, a.status, a.wait_ns);
}

// The same for all 32 lanes of a warp, with one answer for the warp.
__device__ __forceinline__ bool waitw(const GemmArgs &a, int *abort, uint64_t *bar,
                                      uint32_t parity) {
    const bool ok = wait1(a, abort, bar, parity);
    return __all_sync(0xFFFFFFFFu, ok);
}

// ---------------------------------------------------------------- fp16 pair helpers

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
__device__ __forceinline__ __half2 u2h(uint32_t v) { return *reinterpret_cast<__half2 *>(&v); }
__device__ __forceinline__ uint32_t h2u(__half2 v) { return *reinterpret_cast<uint32_t *>(&v); }

// Row r's 64 operand values of one stage (32 fp16 pairs) into its 128-byte row of a
// 128-byte-swizzled K-major operand atom (chunk c lands at 16-byte position c ^ (r & 7)).
__device__ __forceinline__ void store_row(uint8_t *atom, int r, const uint32_t (&v)[32]) {
    uint8_t *rowbase = atom + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
    for (int c = 0; c < 8; c++)
        *reinterpret_cast<uint4 *>(rowbase + ((c ^ (r & 7)) << 4)) =
            make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

__device__ __forceinline__ float tf32_round(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

// Power-of-two scale of a row whose largest block scale is m: 2^e with m in [2^e, 2^(e+1)),
// 1 for m == 0 (an all-zero or non-finite row).  Returns 2^e; *inv = 2^-e.
__device__ __forceinline__ float row_scale(float m, float *inv) {
    if (!(m > 0.0f)) {
        *inv = 1.0f;
        return 1.0f;
    }
    const int e = (int)((__float_as_uint(m) >> 23) & 0xFF) - 127;   // m is a normal float
    *inv = __uint_as_float((uint32_t)(127 - e) << 23);
    return __uint_as_float((uint32_t)(127 + e) << 23);
}

// silu(g) * u with CUDA's expf and an IEEE division (a few ulp): h feeds the Q8_1 rounding of
// the down projection's input, where an error of 1e-6 already moves roundings that a value
// closer to the exact h keeps.
__device__ __forceinline__ float silu_mul(float g, float u) {
    return __fdiv_rn(g, 1.0f + expf(-g)) * u;
}

// Q8_1 of one token's 32 values of h held one per lane (the quantizer of the rest of the
// library: d = amax / 127, q = round-half-away(h / d) clamped to 127), written in the Q8_1(h)
// layout of the workspace.  For normal d the product h * RN(1/d) is within 2 ulp of RN(h / d),
// and |h / d| <= 127 makes 2 ulp < 2^-15: unless the product lies that close to a half-integer
// both round to the same integer; those rare cases, and a subnormal d, take the IEEE division.
__device__ __forceinline__ void quantize_h_lane(const GemmArgs &a, float v, int slot, int f) {
    const int lane = threadIdx.x & 31;
    const bool fin = __all_sync(0xFFFFFFFFu, isfinite(v));
    const float amax = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(fabsf(v))));
    const float d = __fdiv_rn(amax, 127.0f);
    int q = 0;
    if (fin && d != 0.0f) {
        const float inv = __frcp_rn(d);
        const float r = v * inv;
        const float ar = fabsf(r);
        const bool near_tie = !(d >= 0x1p-125f) || fabsf(ar - floorf(ar) - 0.5f) < 0x1p-15f;
        const float rq = near_tie ? __fdiv_rn(v, d) : r;
        q = max(-127, min(127, (int)roundf(rq)));
    }
    const int sum = __reduce_add_sync(0xFFFFFFFFu, q);
    const int hb = a.hpad / 32;
    a.hq[(size_t)slot * a.hpad + f] = (int8_t)q;
    if (a.h) a.h[(size_t)slot * a.F + f] = v;
    if (lane == 0) {
        const size_t bi = (size_t)slot * hb + f / 32;
        if (fin) {
            const __half dh = __float2half_rn(d);
            a.hd[bi] = __half_as_ushort(dh);
            a.hs[bi] = __half_as_ushort(__float2half_rn(__fmul_rn(d, (float)sum)));
            a.hsum[bi] = __fmul_rn(__half2float(dh), (float)sum);
        } else {
            a.hd[bi] = 0;
            a.hs[bi] = 0;
            a.hsum[bi] = 0.0f;
            set_status(a.status, MOE_ERR_NONFINITE);
        }
    }
}

}  // namespace tcp
}  // namespace moe
