// ds4moe_internal.cuh -- device layout, launch parameters and small PTX helpers
// shared by the ds4moe kernels (sm_100a).
//
// Device layout of the quantized experts ("row-block tiled"): a matrix of R
// rows and C columns is cut into 32-row blocks; inside a block the 16-byte
// pieces covering 64 consecutive columns of each row are stored for all 32
// rows back to back, so one warp (lane = row) reads 512 contiguous bytes per
// 64-column step.  Per matrix:
//   IQ2 payload  [R/32][C/64][32][16 B]   the two 8-byte groups of columns
//                                        64kt..64kt+63 (grid indices + S word,
//                                        S in the device order below)
//   IQ2 d        [R/32][C/256][32] binary16
//   Q2 codes     [R/32][C/64][32][16 B]  64 two-bit codes, canonical bit order
//   Q2 scales    [R/32][C/64][32][4 B]   the 4 scale/min bytes of those codes
//   Q2 d,dmin    [R/32][NSB][32][2 x binary16], NSB = max(1, C/256): the pair
//                of the superblock holding column 256*sb of the row
// The algorithmic bytes equal the canonical blocks' bytes (66 and 84 per 256
// weights) except that a C < 256 matrix stores its (d, dmin) once per row.
// Q4 layout (layers with 4-bit experts), per matrix:
//   Q4 codes     [R/32][C/64][32][32 B]  64 four-bit codes in the code order
//                                        below
//   Q4 scales    [R/32][C/64][32][4 B]   sc of the 32-weight sub-blocks 2j, 2j+1
//                                        of the 64 columns, then their m
//   Q4 d,dmin    [R/32][C/256][32][2 x binary16]
// (148 bytes per 256 weights against the block's 144: the 6-bit fields are
// kept as bytes).
// Q4 code order: nibble i of word h of lane t (byte 8t + 4h + i/2 of a row's
// 64-column step) holds the code of column q4_dev_col(mode, t, h, i).
//   mode 0 (gate, up; int8 m16n8k32 fragments): word h is the 32-column half
//     h; its low nibbles (i even) are columns 8t + i/2, the high nibbles
//     columns 8t + 4 + i/2 -- one mask gives the A register of columns
//     8t..8t+3, a shift and the mask that of 8t+4..8t+7.
//   mode 1 (down; bf16 m16n8k16 fragments over the routed h layout, where
//     lane t's four values of a 16-column group are its columns t, 4+t, 8+t,
//     12+t): word h covers the 16-column groups 2h, 2h+1; nibbles (p, p+4)
//     are columns 16 (2h + p/2) + 8 (p & 1) + t + {0, 4}, so that one shift
//     and mask of the word lands both codes in a bf16 pair's mantissas.
//   (q4_dev_col below.)
// Shared (bf16) matrices are stored in 8x8 core-matrix tiles:
//   [R/8][C/8][8 rows][8 cols], 128 contiguous bytes per tile.
// IQ2 S word, device order: byte c (c = 0..3) holds the seven stored signs of
// chunk c in bits 0..6 and bit c of the 4-bit group scale in bit 7 (the block
// keeps the signs at bits 7c..7c+6 and the scale at bits 28..31).  One byte
// per chunk lets a byte-permute place a chunk's signs in a table address.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ds4 {

constexpr int kQK = 256;

// IQ2 S word: block order -> device order, and the fields of the device order.
__host__ __device__ __forceinline__ uint32_t iq2_s_to_device(uint32_t S) {
    uint32_t o = 0;
    for (int c = 0; c < 4; ++c) o |= (((S >> (7 * c)) & 127u) | (((S >> (28 + c)) & 1u) << 7)) << (8 * c);
    return o;
}
__host__ __device__ __forceinline__ uint32_t iq2_dev_scale(uint32_t Sd) {
    return ((Sd >> 7) & 1u) | ((Sd >> 14) & 2u) | ((Sd >> 21) & 4u) | ((Sd >> 28) & 8u);
}
__host__ __device__ __forceinline__ uint32_t iq2_dev_signs(uint32_t Sd, int c) { return (Sd >> (8 * c)) & 127u; }
constexpr int kQ2Bytes = 84;
constexpr int kQ4Bytes = 144;

// Column (0..63, within a 64-column step) of the Q4 code at nibble i of word
// h of lane t, for the gate/up (mode 0) and down (mode 1) code orders.
__host__ __device__ __forceinline__ int q4_dev_col(int mode, int t, int h, int i) {
    if (mode == 0) return 32 * h + 8 * t + 4 * (i & 1) + (i >> 1);
    const int p = i & 3, e = i >> 2;
    return 32 * h + 16 * (p >> 1) + 8 * (p & 1) + 4 * e + t;
}

constexpr int kIQ2Bytes = 66;

enum : uint32_t { kErrBounds = 1u, kErrTimeout = 2u, kErrGrid = 4u };

// Pointers into the caller's weight buffer, in the layout above.
struct Weights {
    const uint8_t* grid_u8;     // [256][8]
    const uint32_t* gtab;       // decode tables of the grid, made by set_grid: [256] magnitude classes of each
                                // row (nibble i = class of element i), [128] sign nibbles of each 7-bit sign
                                // field (bit 2 of nibble i; element 7 from the parity), then the four
                                // magnitudes as int8, their negatives, refused (0/1), distinct values
    const uint32_t* gtab_rows;  // the decode kernel's shared-memory selector table for one or two tokens
                                // ([256][64] words: row r holds class word r in lanes 0..31 and sign word
                                // r & 127 in lanes 32..63), made by set_grid, copied in with one bulk copy
    const float* W_r;           // [E][H]
    const float* W_r2;          // [ceil(E/2)][H][2]: expert pairs interleaved per column (prefill plan), or nullptr
    const float* b_r;           // [E] or nullptr
    const uint8_t* gate_qs;     // IQ2 payload, expert stride iq2_qs_stride bytes
    const uint16_t* gate_d;     // IQ2 d, expert stride iq2_d_stride elements
    const uint8_t* up_qs;
    const uint16_t* up_d;
    const uint8_t* down_q;      // Q2 codes, expert stride q2_q_stride bytes
    const uint32_t* down_sc;    // Q2 scales, expert stride q2_sc_stride words
    const uint32_t* down_dd;    // Q2 (d, dmin), expert stride q2_dd_stride words
    const __nv_bfloat16* sh_gate;   // [I/8][H/8][8][8]
    const __nv_bfloat16* sh_up;
    const __nv_bfloat16* sh_down;   // [H/8][I/8][8][8]
    size_t iq2_qs_stride, iq2_d_stride, q2_q_stride, q2_sc_stride, q2_dd_stride;
    // Q4 layout (expert_bits 4): codes in gate_qs / up_qs / down_q, expert stride q4_q_stride bytes; scale
    // words and (d, dmin) words below, expert strides q4_sc_stride / q4_dd_stride words (gate and up share
    // the strides; down's shape is the transpose, same sizes)
    const uint32_t* gate_sc4;
    const uint32_t* up_sc4;
    const uint32_t* down_sc4;
    const uint32_t* gate_dd4;
    const uint32_t* up_dd4;
    const uint32_t* down_dd4;
    size_t q4_q_stride, q4_sc_stride, q4_dd_stride;
};

struct Dims {
    int H, I, E, k;
    int has_shared;
    int act_bf16;
    int q4;                     // routed experts in the Q4 layout (all three matrices)
};

// Workspace pointers (decode plan).
struct DecodeWs {
    uint32_t* err;          // device error word
    uint32_t* ticket;       // router last-CTA ticket
    uint32_t* queue;        // projection task counter (one token: shared-expert gate/up tasks, then down tasks)
    uint32_t* queue_rt;     // one token: the routed gate/up task counter
    uint32_t* done;         // projection CTAs finished (the last one resets the counters)
    uint32_t* grid_refused; // this call's projection grid refused the grid (too many or too large magnitudes): 1, else 0
    uint32_t* route_ready;  // set by the router once ids / weights are written; reset by the projection grid
    uint32_t* gu_done;      // gate/up tasks finished, h stored: [0] shared (of I/8), [1 + u] routed entry u
                            //   (of I/32); the down tasks wait on them; the last CTA resets them
    float* logits;          // [n][E]
    int32_t* ids;           // [n][k]
    float* wts;             // [n][k]
    uint16_t* hb_rt;        // [n*k][I/64][2][64] bf16: h of each routed slot as two pieces (hi, lo = h - hi);
                            //   inside each 16-column block position 4c + e holds column c + 4e
    float* hsum_rt;         // [n*k][I/16]: per 16-column block, the sum of hi + lo
    uint16_t* hb_sh;        // [n][I/64][2][64] bf16: h of the shared expert as two pieces, natural order
    float* y_rt;            // [n*k][H]
    float* y_sh;            // [n][H]
    const void* xres;       // x again when the call adds the residual (out = x + layer(x)), else nullptr
    const float* steer_v;   // [H] steering direction, or nullptr (no steering)
    float steer_F;          // steering strength: y -= F v (v . y)
    int stages;             // projections run: 1 gate and up, 2 down, 3 both (the forward)
    int probe;              // 0: forward; 1: every token to routed expert probe_e; 2: the shared expert alone
    int probe_e;
    float* probe_out;       // probe: raw accumulators (gate/up: [n][2I]; down: [n][H])
    // chained forward (ds4moe_forward_chain): the combine CTAs add 1 to chain_done once out is written;
    // the next layer's projection prologue waits until chain_wait (the previous layer's chain_done)
    // reaches chain_target, and its last CTA resets that counter
    uint32_t* chain_done;
    uint32_t* chain_wait;
    uint32_t chain_target;
};

// Caller routing (ds4moe_forward_routed): ids_in / wts_in [nslots] copied to
// ids / wts; an id outside [0, E) becomes expert 0 with weight 0 and sets
// kErrBounds.  With `ready`, one CTA, which publishes the routing through it
// (release) once every slot is written.
__global__ void k_routing_in(const int32_t* ids_in, const float* wts_in, int nslots, int E, int32_t* ids, float* wts,
                             uint32_t* ready, uint32_t* err);

// Workspace pointers (prefill plan).
struct PrefillWs {
    float* logits;          // [n][E]
    int32_t* ids;           // [n][k]
    float* wts;             // [n][k]
    int32_t* blk_cnt;       // [blocks of 1024 slots][E]
    int32_t* blk_off;       // [blocks][E]
    int32_t* counts;        // [E] slots per expert
    int32_t* offs;          // [E + 1] first position of each expert
    int32_t* mt_prefix;     // [E + 1] 128-row tiles before each expert
    int32_t* pos_of_slot;   // [n k]
    int32_t* slot_of_pos;   // [n k]
    __nv_bfloat16* xb;      // [n][H] x in bf16 (binary32 activations only)
    __nv_bfloat16* Xp;      // [n k][H] permuted activations
    __nv_bfloat16* Hb;      // [n k][I] routed h
    __nv_bfloat16* Hs;      // [n][I] shared h
    float* Y;               // [n k][H] routed outputs (unweighted)
    float* Ys;              // [n][H] shared output
    uint32_t* err;
    uint32_t* grid_refused; // this call's routed GEMMs refused the grid (more than four magnitudes): 1, else 0
    const void* xres;       // x again when the call adds the residual (out = x + layer(x)), else nullptr
    const float* steer_v;   // [H] steering direction, or nullptr (no steering)
    float steer_F;          // steering strength: y -= F v (v . y)
};

// ---------------------------------------------------------------- helpers
// Sum of one float per thread over a CTA of NT threads in a fixed order
// (butterfly in each warp, then the warp sums in warp order); every thread
// gets the result.  red: NT / 32 floats of shared memory.
template <int NT>
__device__ __forceinline__ float cta_sum_fixed(float v, float* red) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    const int warp = threadIdx.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) s += red[w];
    return s;
}

// Element i of an activation array (binary32, or bf16 widened exactly).
__device__ __forceinline__ float act_at(const void* x, int64_t i, int act_bf16) {
    return act_bf16 ? __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(x) + i) << 16)
                    : __ldg(reinterpret_cast<const float*>(x) + i);
}

__device__ __forceinline__ float half_bits(uint32_t b) { return __half2float(__ushort_as_half((unsigned short)b)); }

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// The same with an L2 cache policy (e.g. evict_last for data that other CTAs read again soon).
__device__ __forceinline__ uint4 ld_stream_v4_hint(const void* p, uint64_t pol) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p), "l"(pol));
    return v;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
    uint2 v;
    asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
    uint32_t v;
    asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream_u16(const void* p) {
    unsigned short v;
    asm("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// One 32-byte global store (sm_100 256-bit vector store).
__device__ __forceinline__ void st_global_v8(void* p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t a4,
                                             uint32_t a5, uint32_t a6, uint32_t a7) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a0), "r"(a1), "r"(a2), "r"(a3),
                 "r"(a4), "r"(a5), "r"(a6), "r"(a7)
                 : "memory");
}

// Packed binary32 pair multiply (sm_100): d = a * b elementwise.
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    unsigned long long A, B, D;
    A = *reinterpret_cast<unsigned long long*>(&a);
    B = *reinterpret_cast<unsigned long long*>(&b);
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(A), "l"(B));
    return *reinterpret_cast<float2*>(&D);
}

// Packed binary32 pair add (sm_100): d = a + b elementwise.
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    unsigned long long A, B, D;
    A = *reinterpret_cast<unsigned long long*>(&a);
    B = *reinterpret_cast<unsigned long long*>(&b);
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(A), "l"(B));
    return *reinterpret_cast<float2*>(&D);
}

// Packed binary32 pair FMA (sm_100): d = a * b + c elementwise.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long A, B, C, D;
    A = *reinterpret_cast<unsigned long long*>(&a);
    B = *reinterpret_cast<unsigned long long*>(&b);
    C = *reinterpret_cast<unsigned long long*>(&c);
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(D) : "l"(A), "l"(B), "l"(C));
    return *reinterpret_cast<float2*>(&D);
}

__device__ __forceinline__ void set_err(uint32_t* err, uint32_t bit) { atomicOr(err, bit); }

// ---------------------------------------------------------------- async copies
// Shared-memory address of a generic pointer (for mbarrier / bulk-copy operands).
__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (bulk-copy) unit.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with `parity` of `bar`, giving up after kWaitNs: the
// error word records the timeout and the caller carries on (the results are
// then wrong, but the kernel ends and the context stays usable).
constexpr uint64_t kWaitNs = 500ull * 1000 * 1000;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > kWaitNs) {
            set_err(err, kErrTimeout);
            return false;
        }
    }
    return true;
}

// Bulk copy global -> shared (16-byte aligned, multiple of 16 bytes), completing
// `bytes` of transaction count on `bar`; L2 policy: evict first (read once).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// Bulk copy global -> shared without an L2 policy (data just written by the
// previous grid).
__device__ __forceinline__ void bulk_load_plain(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// L2 prefetch of bytes at p (16-byte aligned, a multiple of 16 bytes); no completion to wait for.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Part `part` of `nparts` of a region (16-byte aligned start) prefetched into L2 in pieces of at most
// 64 KB; the parts are 256-byte aligned and the region's last partial 16 bytes are left out.
__device__ inline void prefetch_share(const void* base, size_t bytes, int part, int nparts) {
    const size_t per = ((bytes + nparts - 1) / nparts + 255) & ~(size_t)255;
    const size_t lo = (size_t)part * per;
    if (lo >= bytes) return;
    const size_t hi = (lo + per < bytes ? lo + per : bytes) & ~(size_t)15;
    for (size_t o = lo; o < hi; o += 65536)
        prefetch_l2(static_cast<const unsigned char*>(base) + o, (uint32_t)(hi - o < 65536 ? hi - o : 65536));
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Programmatic dependent launch: wait for the preceding grid's results /
// allow the following grid to start.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Barrier among the `nthreads` threads (whole warps) that use barrier `id`.
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// silu(z) = z / (1 + e^-z) with the fast exponential and reciprocal (relative
// error a few ulp of binary32; e^-z = inf gives -0 or 0, the limit).
__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

}  // namespace ds4
