/*
 * moe.h -- C ABI of libmoe.so, a B200 (sm_100a) quantized mixture-of-experts layer.
 *
 * The layer (the per-token expert path of the Strata engine pages):
 *   - "Strata: a 125B MoE at 94 tok/s on a 12 GB Card", section "Three architecture facts":
 *     512 experts per layer, 10 routed + 1 always-on shared expert, hidden size 2,560;
 *     "Strata-Sage-A1.5-GGUF": 256 experts, top-8.
 *   - "Strata v0.1.31" release notes, section "Experimental: Unsloth UD-Q4_K_XL on a normal
 *     PC": experts stored as Q4_K, Q5_K, Q5_1 and Q8_0 blocks (GGUF), decoded bit for bit as
 *     llama.cpp decodes them, dot products equal to ggml's within float rounding.
 *   - "Strata v0.1.39" release notes, fixes list, #606: q8_1 activations;
 *     "Strata-Sage-A1.5-GGUF", round-2 table: one activation quantization per token.
 *
 * For a batch of T tokens:  x fp32 [T][H], router logits fp32 [T][E]  ->  out fp32 [T][H]
 *   a1  x is quantized once per token to Q8_1 blocks of 32 (int8 q, fp16 d, fp16 s)
 *   a2  each token takes its k largest logits (ties: lower expert id) with weights
 *       w = softmax over those k logits
 *   a3  (token, slot) pairs are grouped by expert: counts, exclusive offsets, a permutation
 *       stable in token order
 *   a4  every chosen expert computes g = W_gate x^, u = W_up x^ from its packed weights
 *   a5  h = silu(g) * u, re-quantized to Q8_1
 *   a6  y = W_down h^
 *   a7  out[t] = sum_j w[t][j] * y[t][e_j] + y[t][shared]     (shared expert: weight 1)
 *
 * Conventions for every entry point:
 *   - Pointers named d_* are DEVICE pointers (cudaMalloc / torch CUDA memory) of the current
 *     device; host_* are host pointers.  The caller owns all memory passed in.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *   - Work is enqueued asynchronously; MOE_OK means "validated and enqueued".
 *   - Argument errors are detected on the host and returned before anything is enqueued.
 *   - Problems only the device can see (a non-finite input, a bounded wait that ran out)
 *     are recorded as the first error code in a 32-bit status word that the caller reads
 *     with moe_read_status.  No kernel traps.
 *   - No C++ exception crosses this interface.  Calls are thread-safe when they use distinct
 *     workspaces.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* bad size, null pointer, k > E, ...                      */
    MOE_ERR_UNSUPPORTED = 2,   /* a shape or format this build does not handle             */
    MOE_ERR_ALIGNMENT = 3,     /* a pointer or row stride not aligned as required          */
    MOE_ERR_CUDA = 4,          /* a CUDA runtime call failed (launch, copy, attribute)     */
    MOE_ERR_NONFINITE = 5,     /* device: an activation block or a logit row was not finite */
    MOE_ERR_BOUNDS = 6,        /* descriptor offsets/strides reach outside the arena       */
    MOE_ERR_TIMEOUT = 7,       /* device: a bounded wait gave up                           */
    MOE_ERR_WORKSPACE = 8      /* workspace smaller than moe_workspace_size reported       */
} moe_status;

/* Block formats of the expert weights (GGUF layouts, little endian):
 *   Q4_K  256 weights in 144 B: fp16 d, fp16 dmin, 12 B of packed 6-bit sub-block scales and
 *         mins (8 sub-blocks of 32), 128 B of 4-bit quants; w = d*sc*q - dmin*m
 *   Q5_K  256 weights in 176 B: as Q4_K plus a 32 B plane of fifth bits before the quants
 *   Q8_0  32 weights in 34 B: fp16 d, 32 int8 q; w = d*q
 *   Q5_1  32 weights in 24 B: fp16 d, fp16 m, 32 fifth bits (uint32), 16 B of 4-bit quants
 *         (element n < 16: low nibble of byte n, n >= 16: high nibble of byte n-16);
 *         w = d*q + m
 *   Q6_K  256 weights in 210 B: 128 B of low 4 bits, 64 B of high 2 bits, 16 int8 scales (one
 *         per 16 weights), fp16 d; w = d*sc*(q - 32).  The format real Q4_K_M model files mix
 *         into their FFN tensors.  Dequant-GEMV and CUDA-core paths only: an arena holding a
 *         Q6_K expert takes no tensor-core plan (its integer products sc*(q-32) reach 12
 *         significant bits; the exact fp16 operands of that path hold 11).                    */
typedef enum {
    MOE_FMT_Q4_K = 0,
    MOE_FMT_Q5_K = 1,
    MOE_FMT_Q8_0 = 2,
    MOE_FMT_Q5_1 = 3,
    MOE_FMT_Q6_K = 4
} moe_fmt;

/* One expert inside the arena.  Matrices follow the GGUF convention: a row is one output
 * neuron, blocks run along the input dimension.  gate and up: ffn rows of `hidden` weights;
 * down: `hidden` rows of `ffn` weights rounded up to whole blocks (the weights past `ffn` must
 * decode to 0).  off[] are byte offsets from the arena base (multiples of 16); stride[] are
 * row strides in bytes (multiples of 16, at least the packed row size).                      */
typedef struct {
    int32_t fmt;          /* moe_fmt */
    int32_t reserved;     /* must be 0 */
    uint64_t off[3];      /* gate, up, down */
    uint64_t stride[3];   /* gate, up, down */
} moe_expert_desc;

typedef struct moe_arena moe_arena;

/* Register a device-resident expert arena: `n_experts` routed experts plus, when
 * shared_expert >= 0, one more descriptor at index n_experts for the always-on shared expert
 * (shared_expert must then equal n_experts).  host_descs has n_experts (+1) entries.
 * hidden: multiple of 256 (K-quants) or 32 (Q8_0 and Q5_1 only); ffn: multiple of 32.
 * Checks every descriptor against arena_bytes (MOE_ERR_BOUNDS) and alignment; copies the table
 * to the device (the one allocation the library makes, freed by moe_arena_destroy).  d_arena
 * (256-byte aligned) must stay valid until moe_arena_destroy.                                */
moe_status moe_arena_create(const void *d_arena, size_t arena_bytes, int hidden, int ffn,
                            int n_experts, int shared_expert, const moe_expert_desc *host_descs,
                            moe_arena **out);
void moe_arena_destroy(moe_arena *arena);

/* Forward flags. */
#define MOE_F_DETERMINISTIC 1u   /* prefill: combine by gathering per-token sums (no atomics) */
#define MOE_F_FORCE_DECODE 2u    /* use the grouped dequant-GEMV path whatever T is          */
#define MOE_F_FORCE_PREFILL 4u   /* use the grouped tensor-core GEMM path whatever T is; the
                                    workspace must be sized with this flag (else
                                    MOE_ERR_WORKSPACE); MOE_ERR_UNSUPPORTED when the arena's
                                    shape has no tensor-core plan (hidden % 256 or ffn % 64)   */
#define MOE_F_KEEP_H 8u          /* also store fp32 h (SwiGLU output) in the workspace       */
#define MOE_F_LOOKAHEAD 16u      /* moe_chain_forward: prefetch the next layer's predicted
                                    experts into L2 while a layer runs (batches of <= 16)    */
#define MOE_F_TC_I8 32u          /* tensor-core path: gate/up as 8-bit integer products
                                    (tcgen05 kind::i8, one s32 accumulator per 32-weight block,
                                    promoted in fp32) instead of exact kind::f16 products     */

/* Bytes of device workspace moe_forward needs for up to max_tokens tokens, k routed experts
 * per token and the given flags.  The workspace is caller-owned scratch, 256-byte aligned. */
moe_status moe_workspace_size(const moe_arena *arena, int max_tokens, int k, uint32_t flags,
                              size_t *bytes);

/* a1 alone.  d_x fp32 [T][H] -> d_q int8 [T][H], d_d / d_s fp16 bits [T][H/32] (SoA: the
 * int8 rows stay contiguous).  H multiple of 32.  d_status (may be NULL): device uint32 that
 * receives MOE_ERR_NONFINITE if a block held a non-finite value (that block is written as
 * q = 0, d = s = 0).  All pointers 16-byte aligned.                                          */
moe_status moe_quantize_act(const float *d_x, int T, int H, int8_t *d_q, uint16_t *d_d,
                            uint16_t *d_s, uint32_t *d_status, void *stream);

/* The router: d_logits fp32 [T][E] = d_x fp32 [T][H] times d_router fp32 [E][H] (row e holds
 * expert e's weights), each logit summed in fp32 in a fixed order.  The pages keep the routers
 * on the GPU in the per-token path ("Strata: a 125B MoE at 94 tok/s on a 12 GB Card", "Three
 * architecture facts").  H multiple of 4; d_x and d_router 16-byte aligned, d_logits 4-byte
 * aligned.  Returns MOE_ERR_INVALID_ARG / MOE_ERR_ALIGNMENT before enqueueing anything.      */
moe_status moe_router_logits(const float *d_x, int T, int H, const float *d_router, int E,
                             float *d_logits, void *stream);

/* An optional gate on the shared expert: d_gate fp32 [T] = 1 / (1 + exp(-x[t] . gate_row)),
 * from d_x fp32 [T][H] and d_gate_row fp32 [H].  The pages describe no such gate; models of
 * the Qwen-Next family scale their shared expert by it.  Same argument rules as
 * moe_router_logits.                                                                         */
moe_status moe_shared_gate(const float *d_x, int T, int H, const float *d_gate_row,
                           float *d_gate, void *stream);

/* Bytes of workspace moe_route_topk needs for T tokens, E experts, k per token. */
moe_status moe_route_workspace_size(int T, int E, int k, size_t *bytes);

/* a2 + a3 alone.  d_logits fp32 [T][E] -> d_ids int32 [T][k] (descending logit, ties to the
 * lower id), d_w fp32 [T][k] (softmax over the chosen logits), d_counts int32 [E],
 * d_offsets int32 [E+1] (exclusive prefix sum), d_perm int32 [T*k]: perm[offsets[e] + r] =
 * t*k + j for the r-th pair routed to e in ascending t; d_inv_perm (may be NULL) int32
 * [T*k].  1 <= k <= min(E, 32), E <= 4096.  A token whose logits are not all finite gets ids
 * 0..k-1, weights 1/k and MOE_ERR_NONFINITE in d_status (may be NULL).                       */
moe_status moe_route_topk(const float *d_logits, int T, int E, int k, int32_t *d_ids,
                          float *d_w, int32_t *d_counts, int32_t *d_offsets, int32_t *d_perm,
                          int32_t *d_inv_perm, uint32_t *d_status, void *d_ws, size_t ws_bytes,
                          void *stream);

/* The whole layer, a1-a7.  d_x fp32 [T][hidden], d_logits fp32 [T][n_experts] -> d_out fp32
 * [T][hidden] (overwritten).  1 <= T <= the max_tokens the workspace was sized for,
 * 1 <= k <= min(n_experts, 32).  Intermediates (Q8_1 of x, ids, w, counts, offsets, perm,
 * Q8_1 of h, optional fp32 h) are left in the workspace; moe_ws_views locates them.  They
 * equal what moe_quantize_act / moe_route_topk produce for the same inputs.
 * The grouped dequant-GEMV path (decode) is taken for T <= 16 unless a FORCE flag says
 * otherwise; larger batches take the tensor-core path when the arena allows it (hidden a
 * multiple of 256, ffn a multiple of 64, stored weights and Q8_1 values of magnitude below
 * 65504, which fp16 operands hold) and CUDA-core grouped kernels otherwise (or with
 * MOE_F_FORCE_DECODE).  The decode kernel is one persistent CTA per SM whose CTAs wait for
 * one another (bounded): it needs every SM free for the duration of the call; if other work
 * keeps SMs busy the wait gives up after the arena's wait limit with MOE_ERR_TIMEOUT in the
 * status word.  The workspace's status word collects device-side errors (moe_read_status).  */
moe_status moe_forward(const moe_arena *arena, const float *d_x, const float *d_logits, int T,
                       int k, float *d_out, void *d_ws, size_t ws_bytes, uint32_t flags,
                       void *stream);

/* Device addresses of the intermediates inside a workspace laid out for (T, k, flags).
 * Q8_1 of h is stored per slot: slot s < T*k is the s-th entry of perm (grouped by expert),
 * slot T*k + t is token t's shared-expert row.  hpad = ffn rounded up to 256.                */
typedef struct {
    uint32_t *status;          /* 1 word                                               */
    int8_t *xq;                /* [T][hidden]                                          */
    uint16_t *xd, *xs;         /* [T][hidden/32] fp16 bits                             */
    int32_t *ids;              /* [T][k]                                               */
    float *w;                  /* [T][k]                                               */
    int32_t *counts;           /* [E]                                                  */
    int32_t *offsets;          /* [E+1]                                                */
    int32_t *perm, *inv_perm;  /* [T*k]                                                */
    int8_t *hq;                /* [slots][hpad]                                        */
    uint16_t *hd, *hs;         /* [slots][hpad/32] fp16 bits                           */
    float *h;                  /* [slots][ffn] fp32 (MOE_F_KEEP_H only, else NULL)     */
    int32_t slots, hpad;
    uint32_t *counters;        /* 4 words: the decode kernel's grid-wide counters (zero
                                  between calls; diagnostics and failure tests only)     */
} moe_ws_view;

moe_status moe_ws_views(const moe_arena *arena, void *d_ws, int T, int k, uint32_t flags,
                        moe_ws_view *out);

/* Read the workspace's status word (blocks on `stream`), then reset it to 0 when clear != 0.
 * d_status_word: the `status` pointer of moe_ws_views, or any d_status given above.        */
moe_status moe_read_status(uint32_t *d_status_word, void *stream, int clear,
                           moe_status *device_status);

/* Debug export of one matrix (which: 0 gate, 1 up, 2 down; expert n_experts = shared) as
 * fp32 [rows][row weights] where row weights = whole blocks.  Each value is
 * RN32(RN32(d*sc)*q - RN32(dmin*m)) (K-quants), d*q (Q8_0) or RN32(d*q + m) (Q5_1), bit
 * for bit.                                                                                 */
moe_status moe_debug_dequant(const moe_arena *arena, int expert, int which, float *d_out,
                             void *stream);

/* moe_forward without any allocation, for batches of 1..16 tokens.  The pages describe no such
 * call; it exists for callers that may not allocate device memory -- code running under CUDA
 * graph capture, inference loops with a fixed memory budget, plug-ins whose host framework owns
 * every allocation.  Instead of a caller workspace it uses a 4 MiB scratch array compiled into
 * the library (every GPU that loads libmoe.so holds it until the process exits); shapes whose
 * workspace (moe_workspace_size for T, k, flags 0) exceeds 4 MiB return MOE_ERR_UNSUPPORTED.
 * It calls no cudaMalloc/cudaFree: it clears the scratch's status word and counters with
 * cudaMemsetAsync, runs moe_forward on `stream`, and copies the device status word to d_status
 * (device uint32, may be NULL).  The first call on each device looks up the scratch address;
 * make that first call before any stream capture.  All calls share the one scratch area, which
 * keeps the previous call's contents: calls that can overlap on the GPU (different streams,
 * other threads) race and must be serialised by the caller.                                  */
moe_status moe_forward_noalloc(const moe_arena *arena, const float *d_x, const float *d_logits,
                               int T, int k, float *d_out, uint32_t *d_status, void *stream);

/* Kernel timing for profilers and benchmarks.  The three events (cudaEvent_t handles created
 * by the caller, or NULL to stop) are recorded on the stream of every later moe_forward call on
 * this arena that takes the tensor-core path (T > 16 or MOE_F_FORCE_PREFILL): ev_begin just
 * before the gate/up projection kernel, ev_mid just after it, ev_end after the down projection
 * kernel.  cudaEventElapsedTime(ev_begin, ev_mid) is then the gate/up kernel's duration.  The
 * arena keeps the handles (not owned); calls that use them must not overlap.  The pages have
 * no counterpart; it serves the measurement of the grouped GEMM alone.                       */
moe_status moe_set_timing_events(moe_arena *arena, void *ev_begin, void *ev_mid, void *ev_end);

/* Limit, in nanoseconds, of every bounded wait inside the kernels of later calls on this arena
 * (default 2 s).  A wait that runs out ends its kernel with MOE_ERR_TIMEOUT in the status word
 * after the copies it had in flight have landed; the next call starts clean.  The pages'
 * counterpart is the engine's stall watchdog ("Strata - the details", "Troubleshooting").
 * ns > 0; MOE_ERR_INVALID_ARG otherwise.                                                      */
moe_status moe_set_wait_limit(moe_arena *arena, uint64_t ns);

/* The layer with its router and the shared-expert gate in front: the pages keep the routers on
 * the GPU in the per-token path ("Strata: a 125B MoE at 94 tok/s on a 12 GB Card", "Three
 * architecture facts").  One kernel reads d_x once and writes d_logits fp32 [T][n_experts] =
 * x . d_router rows (d_router fp32 [n_experts][hidden], as moe_router_logits) and, when
 * d_gate_row (fp32 [hidden]) is not NULL, d_gate fp32 [T] = 1 / (1 + exp(-x . gate_row)) (as
 * moe_shared_gate); then moe_forward runs on those logits with the shared expert's output
 * scaled by d_gate[t] instead of 1 (a7: out[t] = sum_j w[t][j] y[t][e_j] + g[t] y[t][shared]).
 * d_logits and d_gate are caller-owned outputs, left for inspection.  A gate row on an arena
 * without a shared expert is MOE_ERR_INVALID_ARG.  Workspace, flags and errors as moe_forward;
 * d_router, d_gate_row and d_x 16-byte aligned.                                             */
moe_status moe_forward_routed(const moe_arena *arena, const float *d_x, int T, int k,
                              const float *d_router, const float *d_gate_row, float *d_logits,
                              float *d_gate, float *d_out, void *d_ws, size_t ws_bytes,
                              uint32_t flags, void *stream);

/* A chain of MoE layers on a residual stream, as a decoder runs them ("Strata - the details",
 * "How it works": the verify pass runs the window through every layer).  Each layer reads the
 * RMS-normalised stream, as the MoE block of a pre-norm decoder does.  For each layer l:
 *   xn_l = x_l / sqrt(mean(x_l^2) + MOE_CHAIN_RMS_EPS) * norm_weight (per token; the
 *          layer's RMSNorm weight, 1 when d_norm_weight is NULL),
 *   logits_l = router_l(xn_l), g_l = gate_l(xn_l) (when the layer has a gate row),
 *   out_l = the layer on xn_l (as moe_forward_routed), x_{l+1} = fp32(x_l + out_l);
 * d_x_out fp32 [T][hidden] receives x_L.  Every layer's arena has the same hidden size.  The
 * residual add and the normalisation are folded into the router kernel (one pass over x).
 * MOE_F_LOOKAHEAD (T <= 16): the router kernel of layer l also computes layer l+1's logits on
 * xn_l; layer l's decode kernel takes their top-k (the prediction), and the router kernel of
 * layer l+1 first prefetches the predicted experts' packed rows (and the shared expert's) into
 * L2 from every SM, so that they are on chip when layer l+1 runs -- the engine's router
 * lookahead ("Strata - the details", the STRATA_LOOKAHEAD paragraph), with L2 in place of the
 * engine's VRAM cache.  A wrong prediction costs only bandwidth: layer l+1 always routes on its
 * own logits.
 * Workspace: moe_chain_workspace_size for the same layers, T, k and flags.
 * trace (may be NULL; each pointer in it may be NULL) receives device copies of the
 * intermediates: the layers' inputs and the result, logits, ids, weights, gates, outputs and
 * (MOE_F_LOOKAHEAD) the predicted ids.  The status word of the workspace (moe_chain_status)
 * collects device-side errors of every layer.                                                */
typedef struct {
    const moe_arena *arena;
    const float *d_router;       /* fp32 [n_experts][hidden]                                */
    const float *d_gate_row;     /* fp32 [hidden] or NULL                                   */
    const float *d_norm_weight;  /* fp32 [hidden] or NULL (all ones): the RMSNorm weight    */
} moe_chain_layer;

#define MOE_CHAIN_RMS_EPS 1e-6f

typedef struct {
    float *x;          /* [n_layers + 1][T][hidden]: x_0 .. x_L                              */
    float *xn;         /* [n_layers][T][hidden]: each layer's normalised input xn_l          */
    float *logits;     /* [n_layers][T][max n_experts]: row stride = the largest n_experts  */
    int32_t *ids;      /* [n_layers][T][k]                                                   */
    float *w;          /* [n_layers][T][k]                                                   */
    float *gate;       /* [n_layers][T] (layers without a gate row: left untouched)          */
    float *out;        /* [n_layers][T][hidden]: each layer's output before the residual add */
    int32_t *early;    /* [n_layers][T][k]: entry l >= 1 = layer l's ids predicted from
                          xn_{l-1} (MOE_F_LOOKAHEAD); entry 0 left untouched                 */
} moe_chain_trace;

moe_status moe_chain_workspace_size(const moe_chain_layer *host_layers, int n_layers,
                                    int max_tokens, int k, uint32_t flags, size_t *bytes);
moe_status moe_chain_forward(const moe_chain_layer *host_layers, int n_layers, const float *d_x,
                             int T, int k, float *d_x_out, void *d_ws, size_t ws_bytes,
                             uint32_t flags, const moe_chain_trace *host_trace, void *stream);
/* The status word of a chain workspace (for moe_read_status). */
moe_status moe_chain_status(const moe_chain_layer *host_layers, int n_layers, void *d_ws, int T,
                            int k, uint32_t flags, uint32_t **d_status_word);

/* Number of kernels this library has enqueued (or recorded into a CUDA graph under stream
 * capture) in this process since it was loaded.  Counting a captured forward gives the
 * kernels each replay of that graph launches. */
uint64_t moe_kernels_enqueued(void);

/* Static text of a status code. */
const char *moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
