/*
 * ds4moe.h -- C ABI of the ds4 routed-MoE expert FFN on B200 (sm_100a).
 *
 * The operation (the pages describe the ds4 engine for DeepSeek V4 Flash):
 *   "antirez가 만든 DeepSeek V4 Flash 전용 로컬 추론 엔진 ds4" (jeff.news),
 *   2-bit quantization bullets: only the routed MoE experts are quantized --
 *   up/gate in IQ2_XXS, down in Q2_K -- while the shared experts, the
 *   projections and the routing stay at full precision.
 *   "antirez/ds4 -- Metal용 DeepSeek V4 Flash 로컬 추론 엔진 완벽 가이드"
 *   (sigco.tistory.com), "왜 독자 엔진이 필요할까": each input runs through only
 *   some of the experts.
 * For every token x (length H): router logits l = W_r x (+ b), the top-k
 * experts by (logit desc, index asc), weights w = softmax over those k logits;
 * for each selected expert e: h = silu(W_gate,e x) * (W_up,e x),
 * y_e = W_down,e h; out = y_shared + sum_j w_j y_{e_j}, with the shared expert
 * an unquantized bf16 SwiGLU FFN of the same intermediate size I.
 *
 * Conventions (every function):
 *   - returns ds4moe_status: 0 on success, a negative code otherwise; on an
 *     error nothing is launched and ds4moe_last_error() holds a message.
 *   - pointers named d_* (and every tensor argument unless a function says
 *     "host") are CUDA device pointers owned by the caller; the library never
 *     allocates device memory and never frees the caller's buffers.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All device work is asynchronous on it unless stated.
 *   - matrices are row-major with rows = output features:
 *     W_gate, W_up: [I][H]; W_down: [H][I]; W_r: [E][H].
 *
 * Block formats (little endian; 256 weights per block, blocked over the
 * row-major flat index of the matrix):
 *   Q2_K-style, 84 bytes: [0,16) scale byte j = sc_j | m_j<<4 for sub-block
 *     j (weights 16j..16j+15); [16,80) 2-bit code q_i at byte 16+i/4, bits
 *     2(i%4); [80,82) d, [82,84) dmin as binary16.
 *     weight_i = (d*sc_j)*q_i - dmin*m_j   (one rounding to binary32)
 *   IQ2_XXS-style, 66 bytes: [0,2) d (binary16); eight 8-byte groups g at
 *     2+8g: bytes 0..3 = grid rows a_c of chunks c (8 weights each), bytes
 *     4..7 = uint32 S with sign field sigma_c in bits 7c..7c+6 and the group
 *     scale s_g in bits 28..31.  Element i<7 of chunk c is negative when bit i
 *     of sigma_c is set, element 7 when sigma_c has odd popcount.
 *     weight = d*(2 s_g+1)/8 * G[a_c][i] * (+-1)   (exact in binary32)
 *     G is a 256 x 8 table of uint8 magnitudes supplied by the caller.
 */
#ifndef DS4MOE_H
#define DS4MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DS4MOE_OK = 0,
    DS4MOE_ERR_ARG = -1,        /* NULL pointer, out-of-range count or index */
    DS4MOE_ERR_ALIGN = -2,      /* a pointer is not 16-byte aligned */
    DS4MOE_ERR_SHAPE = -3,      /* unsupported layer shape */
    DS4MOE_ERR_NOT_READY = -4,  /* buffers not bound, or weights not all loaded */
    DS4MOE_ERR_CUDA = -5,       /* a CUDA runtime call failed */
    DS4MOE_ERR_TIMEOUT = -6,    /* a bounded device-side wait gave up */
    DS4MOE_ERR_DEVICE = -7      /* a device-side check failed (see ds4moe_get_device_error) */
} ds4moe_status;

enum { DS4MOE_ACT_F32 = 0, DS4MOE_ACT_BF16 = 1 };

typedef struct {
    int32_t hidden;        /* H: multiple of 256 */
    int32_t inter;         /* I: multiple of 256, or 128 */
    int32_t n_experts;     /* E: 1 .. 1024 */
    int32_t top_k;         /* k: 1 .. min(E, 16) */
    int32_t max_tokens;    /* largest n_tokens any forward call will pass (>= 1) */
    int32_t act_dtype;     /* DS4MOE_ACT_F32 or DS4MOE_ACT_BF16: element type of x */
    int32_t has_shared;    /* 1: add the bf16 shared expert; 0: routed experts only */
    int32_t has_bias;      /* 1: the router adds a bias b[E] */
    int32_t decode_max;    /* n_tokens <= decode_max uses the decode plan
                              (0 selects the default, 8); larger n uses the
                              bf16 tensor-core plan */
    int32_t expert_bits;   /* routed-expert format: 0 or 2 = gate, up IQ2_XXS-
                              style and down Q2_K-style blocks; 4 = all three
                              Q4_K-style blocks (144 bytes per 256 weights:
                              d, dmin binary16; sixteen 6-bit fields (eight
                              scales, eight mins of 32-weight sub-blocks) in
                              the little-endian 96-bit integer of bytes 4..15;
                              the 4-bit code of weight i at byte 16 + i/2, low
                              nibble for even i; weight = d sc q - dmin m).
                              4-bit layers need inter % 256 == 0 and no
                              grid. */
} ds4moe_shape;

typedef struct ds4moe ds4moe_t;   /* opaque handle; host memory owned by the library */

/* Validate the shape and create a handle.  *out receives the handle. */
ds4moe_status ds4moe_create(const ds4moe_shape* shape, ds4moe_t** out);

/* Free the handle (host memory only; bound device buffers stay the caller's). */
ds4moe_status ds4moe_destroy(ds4moe_t* h);

/* Bytes of device memory the caller must provide for the layer weights
 * (router, grid, all experts in the device layout, shared expert). */
size_t ds4moe_weight_bytes(const ds4moe_t* h);

/* Bytes of device scratch a forward of up to n_tokens tokens needs
 * (n_tokens <= max_tokens; pass max_tokens to size one buffer for all). */
size_t ds4moe_workspace_bytes(const ds4moe_t* h, int32_t n_tokens);

/* Bind caller-owned device buffers: d_weights (>= ds4moe_weight_bytes) and
 * d_workspace (>= ds4moe_workspace_bytes(h, max_tokens)), both 256-byte
 * aligned.  Clears the workspace's counters and error word on `stream`.
 * d_workspace may be NULL (with workspace_bytes 0): the weights are bound
 * alone, every call that needs the workspace returns DS4MOE_ERR_NOT_READY,
 * and ds4moe_route_noalloc still works.  Rebinding marks every expert as not
 * loaded. */
ds4moe_status ds4moe_bind(ds4moe_t* h, void* d_weights, size_t weight_bytes, void* d_workspace,
                          size_t workspace_bytes, void* stream);

/* ---- packers (quantizers), on the device -------------------------------- */

/* Quantize n_weights binary32 values d_w (n_weights a multiple of 256, read as
 * consecutive 256-weight blocks of the flat row-major matrix) into Q2_K-style
 * blocks at d_blocks (n_weights/256 * 84 bytes).  Decisions in fp64:
 * per sub-block lo = min(0, min w), hi = max(0, max w), scale = (hi-lo)/3,
 * min = -lo; d = half(max scale/15), dmin = half(max min/15);
 * sc = clamp(rne(scale/d), 0, 15), m = clamp(rne(min/dmin), 0, 15);
 * q = clamp(rne((w + dmin m)/(d sc)), 0, 3); zero divisors give zero fields. */
ds4moe_status ds4moe_pack_q2k(const float* d_w, int64_t n_weights, void* d_blocks, void* stream);

/* Quantize into IQ2_XXS-style blocks (n_weights/256 * 66 bytes) with grid
 * d_grid [256*8] uint8.  Decisions in fp64: d = half(max|w| / (43*31/8))
 * (zero block if d == 0); s_g = clamp(rne(4 max|w_g|/(43 d) - 0.5), 0, 15);
 * per 8-weight chunk the negative flags, with the smallest-|w| element
 * (lowest index on ties) flipped if their count is odd; the grid row
 * minimizing sum (d(2s_g+1)/8 G[a][i] - t_i)^2 over t_i = +-|w_i| (ties to
 * the lowest row). */
ds4moe_status ds4moe_pack_iq2xxs(const float* d_w, int64_t n_weights, const uint8_t* d_grid, void* d_blocks,
                                 void* stream);

/* Quantize into Q4_K-style blocks (n_weights/256 * 144 bytes).  Decisions in
 * fp64, the Q2_K-style rule with 32-weight sub-blocks: per sub-block
 * lo = min(0, min w), hi = max(0, max w), scale = (hi-lo)/15, min = -lo;
 * d = half(max scale/63), dmin = half(max min/63);
 * sc = clamp(rne(scale/d), 0, 63), m = clamp(rne(min/dmin), 0, 63);
 * q = clamp(rne((w + dmin m)/(d sc)), 0, 15); zero divisors give zero fields. */
ds4moe_status ds4moe_pack_q4k(const float* d_w, int64_t n_weights, void* d_blocks, void* stream);

/* ---- loading (device pointers in; repacked into the bound weight buffer) - */

/* Grid magnitudes [256][8] uint8.  The prefill plan (n_tokens > decode_max)
 * expects at most four distinct byte values in the grid (the format's grid
 * uses three); with more, a prefill forward leaves out as it was and records
 * device error bit 2 (see ds4moe_get_device_error); the next forward with a
 * valid grid writes out again. */
ds4moe_status ds4moe_set_grid(ds4moe_t* h, const uint8_t* d_grid, void* stream);

/* Router rows [E][H] binary32 and, when has_bias, bias [E] (else NULL). */
ds4moe_status ds4moe_set_router(ds4moe_t* h, const float* d_W, const float* d_bias, void* stream);

/* Expert e's three matrices as canonical blocks: gate, up IQ2_XXS-style
 * ([I][H] -> I*H/256 blocks), down Q2_K-style ([H][I] -> H*I/256 blocks); for
 * a layer created with expert_bits = 4 all three Q4_K-style (same block
 * counts, 144 bytes each). */
ds4moe_status ds4moe_set_expert(ds4moe_t* h, int32_t e, const void* d_gate, const void* d_up,
                                const void* d_down, void* stream);

/* Shared expert as bfloat16: gate, up [I][H]; down [H][I].  Required when
 * has_shared = 1. */
ds4moe_status ds4moe_set_shared(ds4moe_t* h, const void* d_gate, const void* d_up, const void* d_down,
                                void* stream);

/* Directional steering of the layer output, as the pages' server offers it
 * after the FFN outputs with one binary32 direction vector per layer (the
 * server's option list in the modu-print.com article on ds4.c): every later
 * forward replaces the layer output y (per token, before any residual add) by
 * y - F v (v . y).  d_v: device
 * pointer to H binary32 values, copied on `stream` (the caller may free it
 * afterwards); v . y is summed in a fixed order, so results repeat bitwise.
 * d_v == NULL or F == 0 turns steering off.  Requires hidden <= 4096
 * (DS4MOE_ERR_SHAPE) and a finite F (DS4MOE_ERR_ARG). */
ds4moe_status ds4moe_set_steering(ds4moe_t* h, const float* d_v, float F, void* stream);

/* ---- the hot path -------------------------------------------------------- */

/* out[n_tokens][H] (binary32) = the layer applied to x[n_tokens][H] (element
 * type act_dtype).  x and out are 16-byte aligned device buffers.  Plan:
 * n_tokens <= decode_max -> fp32 GEMV path (router + top-k, fused gate/up +
 * SwiGLU, down + gate-weighted combine); otherwise the bf16 tensor-core path
 * (router, permutation by expert, grouped tcgen05 GEMMs, combine).
 * n_tokens == 0 is a no-op.  Launches only; safe to capture in a CUDA graph. */
ds4moe_status ds4moe_forward(ds4moe_t* h, const void* d_x, int32_t n_tokens, float* d_out, void* stream);

/* out = x + layer(x): the residual step of a chain of layers (one layer's
 * output is the next layer's input, x_{l+1} = x_l + MoE_l(x_l), with no norm
 * in between: the pages' multi-token-prediction verify runs such chains).  The
 * combine kernel adds x (bf16 widened exactly) after the gate-weighted sum, one
 * binary32 add per element.  x and out must not overlap (DS4MOE_ERR_ARG);
 * otherwise as ds4moe_forward. */
ds4moe_status ds4moe_forward_residual(ds4moe_t* h, const void* d_x, int32_t n_tokens, float* d_out, void* stream);

/* The layer with the caller's routing instead of the router's: d_ids
 * [n_tokens][top_k] int32 expert ids and d_w [n_tokens][top_k] binary32
 * weights (device, 4-byte aligned), out[t] = shared(x_t) + sum_j w[t][j]
 * expert_{ids[t][j]}(x_t), j in order, on the plan n_tokens selects.  An id
 * outside [0, n_experts) counts as expert 0 with weight 0 and sets bit 0 of
 * the device error word (ds4moe_get_device_error).  An id may repeat within a
 * token.  The expert step of expert parallelism: a handle over one rank's
 * experts with top_k 1, no shared expert, every received row a token, its
 * local expert id and weight 1, gives each row's expert output. */
ds4moe_status ds4moe_forward_routed(ds4moe_t* h, const void* d_x, int32_t n_tokens, const int32_t* d_ids,
                                    const float* d_w, float* d_out, void* stream);

/* Expert-parallel combine (no handle): out[t][r] = base[t][r] + sum_j
 * w[t][j] y[t k + j][r], j = 0..k-1 in order, one fused multiply-add per slot
 * (the layer's own combine order).  d_y [n k][H], d_w [n][k], d_base [n][H]
 * or NULL (zero), d_out [n][H]: device binary32; d_out may alias d_base. */
ds4moe_status ds4moe_combine_slots(const float* d_y, const float* d_w, const float* d_base, int32_t n, int32_t k,
                                   int32_t hidden, float* d_out, void* stream);

/* A chain of layers on the decode plan: x_{l+1} = x_l + layer_l(x_l) for
 * l = 0 .. n_layers-1 (layers[l] applied to the previous layer's output),
 * x_0 = d_x, the last output to d_out ([n_tokens][hidden] binary32).  The
 * multi-token-prediction verify step of a model whose layers are these
 * handles.  Every handle: bound, loaded, the same hidden size, n_tokens <=
 * its decode_max and max_tokens; layers after the first take binary32 x
 * (act_dtype F32).  d_work: caller device scratch of 2 * n_tokens * hidden
 * binary32 (the intermediate outputs, ping-pong), 16-byte aligned, not
 * overlapping d_x or d_out.  Layer l+1's kernels are launched as programmatic
 * dependents of layer l's: its router loads its rows while layer l's combine
 * runs, and its projection kernel streams the first shared-expert weights
 * before x_{l+1} is ready (its prologue waits, bounded, on a counter that
 * layer l's combine CTAs raise).  Results equal ds4moe_forward_residual layer
 * by layer bit for bit.  Layer handles must be distinct (each keeps its own
 * counters).  Errors as ds4moe_forward; a wait that runs out records
 * DS4MOE_ERR_TIMEOUT in the device error word of the waiting layer. */
ds4moe_status ds4moe_forward_chain(ds4moe_t* const* layers, int32_t n_layers, const void* d_x, int32_t n_tokens,
                                   float* d_out, float* d_work, void* stream);

/* The same computation with HOST buffers: copies x_host to the device (into
 * the workspace), runs ds4moe_forward on `stream`, copies the result to
 * out_host and waits for all of it (ds4moe_forward_host_async followed by
 * ds4moe_host_sync and a synchronize of `stream`).  Pinned host memory gives
 * the fastest copies. */
ds4moe_status ds4moe_forward_host(ds4moe_t* h, const void* x_host, int32_t n_tokens, float* out_host,
                                  void* stream);

/* Pipelined host-buffer forward; returns without waiting.  The workspace holds
 * two staging slots that consecutive calls of a handle alternate between.  A
 * call enqueues (1) the copy of x_host into its slot, on the handle's own
 * upload stream, after the forward that last read that slot; (2) ds4moe_forward
 * on `stream`, after that copy and after the slot's previous result has been
 * copied out; (3) the copy of the result to out_host, on the handle's own
 * download stream, after the forward.  So one call's copies overlap the
 * kernels of its neighbours.  out_host holds the result after
 * ds4moe_host_sync(h); until then x_host must stay unchanged and out_host
 * untouched.  The streams and events are created on the first call (not
 * allowed during stream capture) on the current device and released by
 * ds4moe_destroy.  Errors: as ds4moe_forward; DS4MOE_ERR_CUDA if a copy or
 * an event operation fails.  Not thread-safe per handle. */
ds4moe_status ds4moe_forward_host_async(ds4moe_t* h, const void* x_host, int32_t n_tokens, float* out_host,
                                        void* stream);

/* Waits until every copy enqueued by ds4moe_forward_host_async on h has
 * finished (and with them the forwards they follow).  DS4MOE_OK at once if
 * the handle has made no such call. */
ds4moe_status ds4moe_host_sync(ds4moe_t* h);

/* ---- measurement ---------------------------------------------------------- */

/* Number of kernel launches one ds4moe_forward of n_tokens makes (0 if n_tokens
 * is outside 1..max_tokens). */
int32_t ds4moe_plan_launches(const ds4moe_t* h, int32_t n_tokens);

/* Name of launch i (0-based) of that plan, a static string; NULL if out of range. */
const char* ds4moe_plan_kernel(const ds4moe_t* h, int32_t n_tokens, int32_t i);

/* ds4moe_forward that also records events[2i] on `stream` right before launch
 * i and events[2i+1] right after it, for i < ds4moe_plan_launches(h, n):
 * cudaEvent_t handles created by the caller (with timing enabled).  The
 * elapsed time between the two events of a launch is that kernel's duration
 * on the stream.  Same results as ds4moe_forward. */
ds4moe_status ds4moe_forward_profiled(ds4moe_t* h, const void* d_x, int32_t n_tokens, float* d_out,
                                      void* const* events, void* stream);

/* ds4moe_forward_residual with the same per-launch events. */
ds4moe_status ds4moe_forward_residual_profiled(ds4moe_t* h, const void* d_x, int32_t n_tokens, float* d_out,
                                               void* const* events, void* stream);

/* ---- inspection hooks (same device code as the hot path) ----------------- */

/* Routing only: ids[n][k] (int32, rank order) and weights[n][k] (binary32). */
ds4moe_status ds4moe_route(ds4moe_t* h, const void* d_x, int32_t n_tokens, int32_t* d_ids, float* d_weights,
                           void* stream);

/* Dequantize expert e's matrix `which` (0 gate, 1 up, 2 down) from the
 * loaded device layout into d_out, row-major, as binary32 (as_bf16 = 0) or
 * bfloat16 rounded to nearest even (as_bf16 = 1): the weights the block
 * format defines, read back from the device layout by a plain per-element
 * kernel (a check of the layout and the repack; the hot-path kernels keep
 * their own operand forms, e.g. 1 + q/4 with an affine correction, and
 * ds4moe_probe shows that what they multiply equals these values). */
ds4moe_status ds4moe_dequant(ds4moe_t* h, int32_t e, int32_t which, int32_t as_bf16, void* d_out,
                             void* stream);

/* The grouped-GEMM kernels of a plan run on caller rows, all of them routed to
 * expert e (0..E-1; -1 = the shared expert), with the accumulators written
 * out as they are: the inspection the bit-exactness of the weights the
 * kernels multiply rests on (one-hot rows give back columns of the weight
 * matrices exactly as the tensor cores consumed them).
 *   plan 0 (the decode plan; n <= decode_max): the persistent projection
 *     kernel (gate/up or down tasks only).  which 0: d_in = activations [n][H] binary32 (or bf16
 *     when act_dtype is DS4MOE_ACT_BF16), d_out = [n][2I] binary32, gate
 *     results then up results (no SwiGLU); which 2: d_in = h [n][I]
 *     binary32 (entering as the kernel's two bf16 pieces), d_out = [n][H].
 *   plan 1 (the prefill plan; needs max_tokens > decode_max): the tcgen05
 *     grouped GEMM.  which 0: d_in = activations [n][H] bfloat16, d_out =
 *     [n][2I] binary32, gate accumulators then up accumulators (no SwiGLU);
 *     which 2: d_in = h [n][I] bfloat16, d_out = [n][H] binary32.
 * d_in and d_out are 16-byte aligned device buffers; n in 1..2^20 (plan 1).
 * Uses the workspace of the plan (its routing and intermediates are
 * overwritten). */
ds4moe_status ds4moe_probe(ds4moe_t* h, int32_t plan, int32_t which, int32_t e, const void* d_in, int32_t n_rows,
                           float* d_out, void* stream);

/* The prefill plan's permutation of (token, slot) pairs by expert, on caller
 * ids [n][k] (int32, each in 0..E-1): d_counts [E] slots per expert,
 * d_offsets [E+1] exclusive prefix of the counts, d_pos_of_slot [n*k] the
 * position of slot t*k + j in the permuted order -- a stable counting sort
 * (slots of one expert keep their slot order).  The same kernels the prefill
 * forward runs; needs max_tokens > decode_max and 1 <= n <= max_tokens.
 * Ids outside 0..E-1 are the caller's error (not checked on the device). */
ds4moe_status ds4moe_permutation(ds4moe_t* h, const int32_t* d_ids, int32_t n_tokens, int32_t* d_counts,
                                 int32_t* d_offsets, int32_t* d_pos_of_slot, void* stream);

/* ---- routing without device allocation ------------------------------------ */

/* ds4moe_route for callers that cannot allocate device memory: hosts that own
 * every device buffer through their own pool (a serving process, an embedded
 * runtime) and hand this library only its inputs and outputs, and code that
 * must not call the allocator because cudaMalloc synchronizes the device and
 * would stall the work in flight.  The pages have no counterpart; this is an
 * interface convenience.
 * The router's scratch (logits of up to 8192 token-expert pairs, i.e.
 * n_tokens * n_experts <= 8192, and a 256-byte header of counters and an
 * error word) lives in one static device array inside the library, which
 * every GPU that loads the library holds until the process exits; the bound
 * workspace is not used, and the handle needs only its weight buffer bound
 * (ds4moe_bind accepts a NULL workspace) with the grid and the router loaded.
 * The caller passes x and the outputs ids[n][k] (int32) and weights[n][k]
 * (binary32), with the same results as ds4moe_route.  Larger n_tokens *
 * n_experts, or n_tokens > decode_max, is rejected with DS4MOE_ERR_ARG.
 * The first call on a device looks up the array's device address with that
 * device current (make that first call before any stream capture).  Every
 * call clears the array's counters and shares the one array: calls that
 * overlap on the GPU (other streams, other threads) race, so serialize them.
 * Device-side failures set the array's error word, which
 * ds4moe_get_device_error reads and clears. */
ds4moe_status ds4moe_route_noalloc(ds4moe_t* h, const void* d_x, int32_t n_tokens, int32_t* d_ids,
                                   float* d_weights, void* stream);

/* Check of the failure path every bounded device-side wait takes: runs one
 * warp whose wait (the routine all the kernels' waits use) is on an mbarrier
 * that nothing arrives at.  The wait gives up after its limit (0.5 s), sets
 * bit 1 of the workspace error word and the kernel returns, so the context
 * stays usable; ds4moe_get_device_error then returns DS4MOE_ERR_TIMEOUT.
 * Needs a bound workspace.  Nothing faults, traps or hangs. */
ds4moe_status ds4moe_selftest_wait(ds4moe_t* h, void* stream);

/* Synchronize `stream`, then read and clear the workspace's device error word
 * (and, when ds4moe_route_noalloc has run on the current device, the error
 * word of its static scratch) into *code (0 = none; bit 0 = an index check
 * failed, bit 1 = a bounded wait timed out, bit 2 = the grid has more than
 * four distinct magnitudes).  Returns DS4MOE_ERR_DEVICE / DS4MOE_ERR_TIMEOUT
 * when set; DS4MOE_ERR_NOT_READY when neither word exists. */
ds4moe_status ds4moe_get_device_error(ds4moe_t* h, void* stream, int32_t* code);

/* Message of the last error on the calling thread ("" if none). */
const char* ds4moe_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DS4MOE_H */
