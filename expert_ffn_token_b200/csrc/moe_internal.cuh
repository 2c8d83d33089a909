// moe_internal.cuh -- shared declarations of the libmoe.so kernels (sm_100a only).
//
// Block formats (GGUF layouts, little endian; see include/moe.h):
//   Q4_K 144 B / 256 weights: [0,2) fp16 d, [2,4) fp16 dmin, [4,16) S: packed 6-bit scales and
//        mins of 8 sub-blocks of 32, [16,144) qs: byte 32c+r holds element 64c+r (low nibble,
//        sub-block 2c) and element 64c+32+r (high nibble, sub-block 2c+1).
//   Q5_K 176 B: as Q4_K with qh[32] at [16,48) and qs at [48,176); bit 2c of qh[r] is the fifth
//        bit of element 64c+r, bit 2c+1 that of element 64c+32+r.
//   Q8_0 34 B / 32 weights: fp16 d, int8 q[32].
//   Q5_1 24 B / 32 weights: fp16 d, fp16 m, uint32 qh (bit n: fifth bit of element n),
//        qs[16]: byte i holds element i (low nibble) and element 16+i (high nibble); w = d*q + m.
//   Q6_K 210 B / 256 weights: ql[128] low 4 bits, qh[64] high 2 bits, int8 sc[16] (one per 16
//        weights), fp16 d at 208; element n (h = n/128, i = n%128, g = i/32, l = i%32): low bits
//        = nibble (g >= 2) of ql[64h + l + 32(g&1)], high bits = bits 2g, 2g+1 of qh[32h + l],
//        w = d*sc[8h + 2g + l/16]*(q - 32).
//   Q8_1 (activations, stored SoA): per 32 values int8 q[32], fp16 d, fp16 s = d * sum(q).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "moe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libmoe is built for sm_100a only"
#endif

namespace moe {

constexpr int kQ = 32;            // Q8_1 / Q8_0 block length and K-quant sub-block length
constexpr int kSB = 256;          // K-quant super-block length
constexpr int kQ4KBytes = 144;
constexpr int kQ5KBytes = 176;
constexpr int kQ80Bytes = 34;
constexpr int kQ51Bytes = 24;
constexpr int kQ6KBytes = 210;
constexpr int kMaxK = 32;         // routed experts per token
constexpr int kMaxE = 4096;       // experts per layer
constexpr int kDecodeMaxT = 16;   // largest batch the dequant-GEMV path takes by default
constexpr int kChunk = 64;        // tokens per histogram chunk in the grouping kernels
constexpr uint32_t kPrefetchPiece = 16384;   // bytes per L2 prefetch instruction (lookahead)

// Q8_0 and Q5_1 carry their scale per 32 weights; the K-quants per 256-weight super-block.
__host__ __device__ inline bool small_block(int fmt) {
    return fmt == MOE_FMT_Q8_0 || fmt == MOE_FMT_Q5_1;
}
__host__ __device__ inline int block_weights(int fmt) { return small_block(fmt) ? 32 : 256; }
__host__ __device__ inline int block_bytes(int fmt) {
    return fmt == MOE_FMT_Q4_K   ? kQ4KBytes
           : fmt == MOE_FMT_Q5_K ? kQ5KBytes
           : fmt == MOE_FMT_Q8_0 ? kQ80Bytes
           : fmt == MOE_FMT_Q6_K ? kQ6KBytes
                                 : kQ51Bytes;
}

// Device copy of one expert (the descriptor with the arena base folded in).
struct ExpertDev {
    const uint8_t *m[3];      // gate, up, down
    uint32_t stride[3];
    int32_t fmt;
    int32_t pad;
};

// One unit of grouped work: an expert and the contiguous run of slots routed to it.
// Slots [slot0, slot0 + n) index the Q8_1(h) rows; routed slots are perm positions, the
// shared expert's slots are T*k + t.
struct Job {
    int32_t expert;
    int32_t slot0;
    int32_t n;
    int32_t shared;           // 1 for the shared expert (slot i is token i, weight gate[i] or 1)
};

struct moe_arena_impl;


// Offsets (bytes) of everything moe_forward keeps in its workspace.
struct WsLayout {
    size_t status, sync, blkcnt, njobs, jobs, xq, xd, xs, xsum, ids, w, counts, offsets, perm,
        inv_perm, chunk_counts, chunk_base, hq, hd, hs, hsum, h, y, total;
    // tensor-core path (absent when tc == 0): fp16 activation rows with their power-of-two
    // scales, per token (gate/up) and per slot (down)
    size_t xh, xl, xsh, xsl, xscale, hh, hscale;
    int slots, hpad, max_jobs, n_chunks, tc, kd;
};

// Workspace layout of one moe_forward call (moe_api.cu).  Without allow_tc the tensor-core
// operands are left out.
WsLayout ws_layout(const moe_arena *A, int T, int k, uint32_t flags, bool allow_tc = true);

// The host checks moe_forward makes on its arguments other than the workspace (null pointers,
// sizes, flag combinations, alignment), before anything is enqueued.
moe_status check_forward_args(const moe_arena *arena, const float *d_x, const float *d_logits,
                              int T, int k, const float *d_out, uint32_t flags);

// ------------------------------------------------------------------ device helpers

__device__ __forceinline__ void set_status(uint32_t *st, uint32_t code) {
    if (st) atomicCAS(st, 0u, code);
}

__device__ __forceinline__ float half_bits_to_float(uint32_t bits16) {
    return __half2float(__ushort_as_half((unsigned short)(bits16 & 0xFFFFu)));
}

// Byte i (0..11) of the packed scale words S0 = bytes 4..7, S1 = 8..11, S2 = 12..15 of a block.
__device__ __forceinline__ uint32_t sbyte(uint32_t s0, uint32_t s1, uint32_t s2, int i) {
    uint32_t w = i < 4 ? s0 : (i < 8 ? s1 : s2);
    return (w >> (8 * (i & 3))) & 0xFFu;
}

// 6-bit scale and min of sub-block j of a K-quant block, from the 12 packed bytes.
__device__ __forceinline__ void kq_scale_min(uint32_t s0, uint32_t s1, uint32_t s2, int j,
                                             int &sc, int &mn) {
    if (j < 4) {
        sc = sbyte(s0, s1, s2, j) & 63;
        mn = sbyte(s0, s1, s2, j + 4) & 63;
    } else {
        uint32_t b = sbyte(s0, s1, s2, j + 4);
        sc = (b & 15) | ((sbyte(s0, s1, s2, j - 4) >> 6) << 4);
        mn = (b >> 4) | ((sbyte(s0, s1, s2, j) >> 6) << 4);
    }
}

// ------------------------------------------------------------------ launchers (host)

// Kernels enqueued (or captured into a graph) by this library in this process.
void note_launches(int n);

// Raise a kernel's dynamic shared memory limit to at least `bytes` on the current device.  The
// attribute is set once per (device, kernel, size) so that launches recorded under stream
// capture make no attribute call.
cudaError_t ensure_smem_impl(const void *kernel, size_t bytes);
template <typename Kernel>
inline cudaError_t ensure_smem(Kernel kernel, size_t bytes) {
    return ensure_smem_impl(reinterpret_cast<const void *>(kernel), bytes);
}

cudaError_t launch_quantize(const float *x, int64_t nblocks, int8_t *q, uint16_t *d, uint16_t *s,
                            float *dsum, uint32_t *status, cudaStream_t st);

cudaError_t launch_route_small(const float *x, const float *logits, int T, int H, int E, int k,
                               int shared, const WsLayout &L, uint8_t *ws, cudaStream_t st);

cudaError_t launch_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w,
                        uint32_t *status, cudaStream_t st);

cudaError_t launch_group(const int32_t *ids, int T, int k, int E, int shared, int32_t *counts,
                         int32_t *offsets, int32_t *perm, int32_t *inv_perm,
                         int32_t *chunk_counts, int32_t *chunk_base, Job *jobs, int32_t *njobs,
                         cudaStream_t st);

// The next layer's expert prediction of a chain of layers (the router lookahead): its router
// logits for this batch [T][E] and where its predicted ids go ([T][k]).
struct Lookahead {
    const float *logits;          // null: no lookahead
    int E;
    int32_t *ids_out;
};

// An L2 prefetch of predicted experts' packed rows: ids [n] (-1: none), the layer's expert
// table, its sizes, and the 16 KB pieces of its largest matrix.
struct ExpertPrefetch {
    const int32_t *ids;           // null: none
    int n, shared;                // shared: also the shared expert (index E)
    const ExpertDev *experts;
    int E, H, F, pmax;
};

struct FfnArgs {
    const ExpertDev *experts;
    const Job *jobs;
    const int32_t *njobs;
    const int32_t *perm;
    const int32_t *inv_perm;
    const float *w;
    const int8_t *xq;
    const uint16_t *xd;
    const float *xsum;
    int8_t *hq;
    uint16_t *hd, *hs;
    float *hsum;
    float *h;              // optional fp32 h
    float *y;              // deterministic prefill: y per slot
    float *out;
    const float *gate;     // optional [T]: weight of the shared expert's output (else 1)
    uint32_t *status;
    int T, k, H, F, hpad, max_jobs, fmt_mask;
    int max_stride01, max_stride2;   // largest gate/up and down row strides in the arena
    uint64_t wait_ns;                // limit of every bounded wait in the kernels
    Lookahead look;                  // the decode kernel's fused lookahead (logits null: none)
};

cudaError_t launch_gateup_gemv(const FfnArgs &a, cudaStream_t st);
cudaError_t launch_down_decode(const FfnArgs &a, cudaStream_t st);
cudaError_t launch_down_grouped(const FfnArgs &a, bool deterministic, cudaStream_t st);
cudaError_t launch_combine(const FfnArgs &a, bool shared, cudaStream_t st);

// The whole layer for small batches in one persistent kernel (k_decode.cu).  Sets *taken to
// false, enqueueing nothing, when the shape does not fit its shared-memory plan.
// *look_fused tells whether a.look (when given) runs inside the kernel (the next layer's
// expert count must fit the kernel's top-k width).
cudaError_t launch_decode_fused(const FfnArgs &a, int E, int shared, const float *x,
                                const float *logits, uint8_t *ws, const WsLayout &L,
                                size_t sync_off, size_t blkcnt_off, bool pdl, cudaStream_t st,
                                bool *taken, bool *look_fused);

// Zero Q8_1(h) (int8 layout) in the padded columns [F, hpad) of every slot.
cudaError_t launch_hpad_zero(const FfnArgs &a, cudaStream_t st);

// ---- tensor-core path for large batches (k_gemm_tc.cu)

// One projection phase: 0 = gate/up over the token rows x^, 1 = down over the slot rows h^.
struct TcPhaseArgs {
    FfnArgs ffn;
    const void *wmaps;          // device array of the experts' weight tensor maps
    int phase, slots, keep_h;
    int i8;                     // gate/up on kind::i8 MMAs (k_gateup_i8) instead of kind::f16
    int Kd;                     // down contraction length: ffn rounded up to 64
    const __half *xh, *xl;      // [T][H] fp16 planes, x^ * 2^-e = hi + lo exactly
    const float *xsh, *xsl;     // [T][H/32] block sums xd * sum(q) * 2^-e, tf32 hi + lo
    const float *xscale;        // [T] 2^e
    const __half *hh;           // [slots][Kd] fp16 rows of Q8_1(h) * 2^-e
    const float *hscale;        // [slots] 2^e
    uint64_t wait_ns;           // limit of every wait inside the kernels
};

// Host encoding of every expert's weight tensor maps into `out` (bytes to copy to the device);
// false when the shape or a map is not supported.
bool tc_build_weight_maps(const uint8_t *d_base, const moe_expert_desc *descs, int n, int H,
                          int F, std::vector<uint8_t> &out);
// Dynamic shared memory the tensor-core kernels need for the formats present ((size_t)-1: no
// plan fits); the gate/up kernel's alone.
size_t tc_smem_bytes(int fmt_mask);
size_t tc_gateup_smem_bytes(int fmt_mask);
// One tensor-core phase (phase 0: k_gateup_tc, phase 1: k_down_tc).
cudaError_t launch_gemm_tc(const TcPhaseArgs &p, cudaStream_t st);
cudaError_t launch_gateup_tc(const TcPhaseArgs &p, int grid, cudaStream_t st);
// The gate/up phase with 8-bit integer products and a promotion per 32-weight block
// (k_gateup_i8.cu), and its shared memory ((size_t)-1: no plan fits).
cudaError_t launch_gateup_i8(const TcPhaseArgs &p, int grid, cudaStream_t st);
size_t tc_gateup_i8_smem_bytes(int fmt_mask);
// a1 per token for the tensor-core path: the Q8_1 blocks (as moe_quantize_act) plus the gate/up
// operand planes, the block sums and 2^e.
cudaError_t launch_quant_rows(const float *x, int T, int H, int8_t *xq, uint16_t *xd,
                              uint16_t *xs, float *xsum, __half *xh, __half *xl, float *xsh,
                              float *xsl, float *xscale, uint32_t *status, cudaStream_t st);
// The down operand of every used slot from its Q8_1(h) blocks.
cudaError_t launch_h_rows(const int8_t *hq, const uint16_t *hd, int slots, int F, int hpad, int Kd,
                          __half *hh, float *hscale, cudaStream_t st);

// ---- router, shared gate, lookahead (k_router.cu)

// One pass over the hidden state for up to three sets of fp32 rows [*][H]: router rows Wr [E]
// -> logits [T][E], lookahead rows Wn [En] -> logits_next [T][En], gate row wg -> gate [T].
// With res, the hidden state is x + res (fp32), also written to x_out when x_out is set.  With
// norm, the rows dotted are the hidden state times 1 / sqrt(mean square + eps), then times gamma
// [H] when given, also written to xn_out when xn_out is set.
struct RouterRowsArgs {
    const float *x, *res;
    float *x_out;
    int norm;
    float eps;
    const float *gamma;
    float *xn_out;
    const float *Wr;
    float *logits;
    const float *Wn;
    float *logits_next;
    const float *wg;
    float *gate;
    int E, En, T, H;
    ExpertPrefetch pf;   // issued by the whole grid before the rows
};
// pdl: launched behind the previous kernel of the stream (programmatic dependent launch); the
// kernel prefetches its rows into L2 before it waits for that kernel.
cudaError_t launch_router_rows(const RouterRowsArgs &a, cudaStream_t st, bool pdl);
// Top-k of logits [T][E] (T <= 16) into ids_out [T][k] (-1 for a row that is not finite).
size_t lookahead_smem_bytes(int E);
cudaError_t launch_lookahead(const float *logits, int T, int E, int k, int32_t *ids_out,
                             cudaStream_t st);
cudaError_t launch_residual(const float *x, const float *res, float *x_out, int T, int H,
                            cudaStream_t st);

cudaError_t launch_dequant(const uint8_t *m, int fmt, int rows, int nblocks, int stride,
                           float *out, cudaStream_t st);

}  // namespace moe
