// ds4moe_internal.cuh -- device layout, launch parameters and small PTX helpers
// shared by the ds4moe kernels (sm_100a).
//
// Device layout of the quantized experts ("row-block tiled"): a matrix of R
// rows and C columns is cut into 32-row blocks; inside a block the 16-byte
// pieces covering 64 consecutive columns of each row are stored for all 32
// rows back to back, so one warp (lane = row) reads 512 contiguous bytes per
// 64-column step.  Per matrix:
//   IQ2 payload  [R/32][C/64][32][16 B]   the two 8-byte groups of columns
//                                        64kt..64kt+63 (grid indices + S word)
//   IQ2 d        [R/32][C/256][32] binary16
//   Q2 codes     [R/32][C/64][32][16 B]  64 two-bit codes, canonical bit order
//   Q2 scales    [R/32][C/64][32][4 B]   the 4 scale/min bytes of those codes
//   Q2 d,dmin    [R/32][NSB][32][2 x binary16], NSB = max(1, C/256): the pair
//                of the superblock holding column 256*sb of the row
// The algorithmic bytes equal the canonical blocks' bytes (66 and 84 per 256
// weights) except that a C < 256 matrix stores its (d, dmin) once per row.
// Shared (bf16) matrices are stored in 8x8 core-matrix tiles:
//   [R/8][C/8][8 rows][8 cols], 128 contiguous bytes per tile.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ds4 {

constexpr int kQK = 256;
constexpr int kQ2Bytes = 84;
constexpr int kIQ2Bytes = 66;

enum : uint32_t { kErrBounds = 1u, kErrTimeout = 2u };

// Pointers into the caller's weight buffer, in the layout above.
struct Weights {
    const uint8_t* grid_u8;     // [256][8]
    const float* W_r;           // [E][H]
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
};

struct Dims {
    int H, I, E, k;
    int has_shared;
    int act_bf16;
};

// Workspace pointers (decode plan).
struct DecodeWs {
    uint32_t* err;          // device error word
    uint32_t* ticket;       // router last-CTA ticket
    uint32_t* queue1;       // gate/up task counter
    uint32_t* queue2;       // down task counter
    float* logits;          // [n][E]
    int32_t* ids;           // [n][k]
    float* wts;             // [n][k]
    float* h_rt;            // [n*k][I]
    float* hsum_rt;         // [n*k][I/16]
    float* h_sh;            // [n][I]
    float* y_rt;            // [n*k][H]
    float* y_sh;            // [n][H]
};

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ float half_bits(uint32_t b) { return __half2float(__ushort_as_half((unsigned short)b)); }

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
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

__device__ __forceinline__ float silu(float z) { return z / (1.0f + __expf(-z)); }

}  // namespace ds4
