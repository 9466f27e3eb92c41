// pack.cu -- device quantizers (canonical blocks) and the repack of canonical
// blocks into the device layout.  Load-time code, not on the hot path.
//
// The quantizers take their decisions in fp64 with explicitly rounded
// operations (no contraction), round-half-to-even, so that the same inputs
// give the same bytes on any IEEE machine that follows the same steps.
#include "ds4moe_internal.cuh"

namespace ds4 {

__device__ __forceinline__ uint16_t to_half_bits(double v) { return __half_as_ushort(__double2half(v)); }
__device__ __forceinline__ double from_half_bits(uint16_t b) { return (double)__half2float(__ushort_as_half(b)); }
__device__ __forceinline__ double clamp_rne(double v, double hi) { return fmin(fmax(rint(v), 0.0), hi); }

// ---------------------------------------------------------------- Q2_K-style
// One thread per 256-weight block.
__global__ void k_pack_q2k(const float* __restrict__ w, int64_t n_blocks, uint8_t* __restrict__ out) {
    int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= n_blocks) return;
    const float* x = w + b * kQK;
    uint8_t blk[kQ2Bytes];
    double scale[16], mn[16], max_scale = 0.0, max_min = 0.0;
    for (int j = 0; j < 16; ++j) {
        double lo = 0.0, hi = 0.0;
        for (int i = 0; i < 16; ++i) {
            double v = (double)x[16 * j + i];
            lo = v < lo ? v : lo;
            hi = v > hi ? v : hi;
        }
        scale[j] = __ddiv_rn(__dsub_rn(hi, lo), 3.0);
        mn[j] = -lo;
        max_scale = scale[j] > max_scale ? scale[j] : max_scale;
        max_min = mn[j] > max_min ? mn[j] : max_min;
    }
    uint16_t dh = to_half_bits(__ddiv_rn(max_scale, 15.0));
    uint16_t mh = to_half_bits(__ddiv_rn(max_min, 15.0));
    double d = from_half_bits(dh), dmin = from_half_bits(mh);
    for (int i = 0; i < kQ2Bytes; ++i) blk[i] = 0;
    for (int j = 0; j < 16; ++j) {
        int sc = d > 0.0 ? (int)clamp_rne(__ddiv_rn(scale[j], d), 15.0) : 0;
        int m = dmin > 0.0 ? (int)clamp_rne(__ddiv_rn(mn[j], dmin), 15.0) : 0;
        blk[j] = (uint8_t)(sc | (m << 4));
        double step = __dmul_rn(d, (double)sc), off = __dmul_rn(dmin, (double)m);
        for (int i = 0; i < 16; ++i) {
            int q = 0;
            if (step > 0.0) q = (int)clamp_rne(__ddiv_rn(__dadd_rn((double)x[16 * j + i], off), step), 3.0);
            int kk = 16 * j + i;
            blk[16 + kk / 4] |= (uint8_t)(q << (2 * (kk % 4)));
        }
    }
    blk[80] = dh & 0xff; blk[81] = dh >> 8;
    blk[82] = mh & 0xff; blk[83] = mh >> 8;
    uint8_t* o = out + b * kQ2Bytes;
    for (int i = 0; i < kQ2Bytes; ++i) o[i] = blk[i];
}

// ---------------------------------------------------------------- Q4_K-style
// 6-bit field f of the little-endian 96-bit integer held in bytes 4..15 of a
// block.
__device__ __forceinline__ void q4_set_field(uint8_t* blk, int f, int v) {
    for (int b = 0; b < 6; ++b) {
        const int bit = 6 * f + b;
        blk[4 + bit / 8] |= (uint8_t)(((v >> b) & 1) << (bit % 8));
    }
}
__device__ __forceinline__ int q4_field(const uint8_t* blk, int f) {
    int v = 0;
    for (int b = 0; b < 6; ++b) {
        const int bit = 6 * f + b;
        v |= ((blk[4 + bit / 8] >> (bit % 8)) & 1) << b;
    }
    return v;
}

// One thread per 256-weight block: eight 32-weight sub-blocks, the Q2_K-style
// rule with 4-bit codes and 6-bit scales and mins.
__global__ void k_pack_q4k(const float* __restrict__ w, int64_t n_blocks, uint8_t* __restrict__ out) {
    int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= n_blocks) return;
    const float* x = w + b * kQK;
    uint8_t blk[kQ4Bytes];
    double scale[8], mn[8], max_scale = 0.0, max_min = 0.0;
    for (int j = 0; j < 8; ++j) {
        double lo = 0.0, hi = 0.0;
        for (int i = 0; i < 32; ++i) {
            const double v = (double)x[32 * j + i];
            lo = v < lo ? v : lo;
            hi = v > hi ? v : hi;
        }
        scale[j] = __ddiv_rn(__dsub_rn(hi, lo), 15.0);
        mn[j] = -lo;
        max_scale = scale[j] > max_scale ? scale[j] : max_scale;
        max_min = mn[j] > max_min ? mn[j] : max_min;
    }
    const uint16_t dh = to_half_bits(__ddiv_rn(max_scale, 63.0));
    const uint16_t mh = to_half_bits(__ddiv_rn(max_min, 63.0));
    const double d = from_half_bits(dh), dmin = from_half_bits(mh);
    for (int i = 0; i < kQ4Bytes; ++i) blk[i] = 0;
    for (int j = 0; j < 8; ++j) {
        const int sc = d > 0.0 ? (int)clamp_rne(__ddiv_rn(scale[j], d), 63.0) : 0;
        const int m = dmin > 0.0 ? (int)clamp_rne(__ddiv_rn(mn[j], dmin), 63.0) : 0;
        q4_set_field(blk, j, sc);
        q4_set_field(blk, 8 + j, m);
        const double step = __dmul_rn(d, (double)sc), off = __dmul_rn(dmin, (double)m);
        for (int i = 0; i < 32; ++i) {
            int q = 0;
            if (step > 0.0) q = (int)clamp_rne(__ddiv_rn(__dadd_rn((double)x[32 * j + i], off), step), 15.0);
            const int kk = 32 * j + i;
            blk[16 + kk / 2] |= (uint8_t)(q << (4 * (kk % 2)));
        }
    }
    blk[0] = dh & 0xff; blk[1] = dh >> 8;
    blk[2] = mh & 0xff; blk[3] = mh >> 8;
    uint8_t* o = out + b * kQ4Bytes;
    for (int i = 0; i < kQ4Bytes; ++i) o[i] = blk[i];
}

// ---------------------------------------------------------------- IQ2_XXS-style
// One warp per 256-weight block; lane = 8-weight chunk (group = lane / 4).
__global__ void k_pack_iq2(const float* __restrict__ w, int64_t n_blocks, const uint8_t* __restrict__ grid,
                           uint8_t* __restrict__ out) {
    __shared__ uint8_t sgrid[256 * 8];
    for (int i = threadIdx.x; i < 256 * 8; i += blockDim.x) sgrid[i] = grid[i];
    __syncthreads();
    int lane = threadIdx.x & 31;
    int64_t b = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (b >= n_blocks) return;
    const float* xc = w + b * kQK + 8 * lane;
    uint8_t* o = out + b * kIQ2Bytes;
    double amax = 0.0;
    for (int i = 0; i < 8; ++i) amax = fmax(amax, fabs((double)xc[i]));
    double cmax = amax;   // this chunk's max|w|
    for (int m = 16; m >= 1; m >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    uint16_t dh = to_half_bits(__ddiv_rn(amax, 166.625));   // 43 * 31 / 8
    double d = from_half_bits(dh);
    if (d == 0.0) {
        for (int i = lane; i < kIQ2Bytes; i += 32) o[i] = 0;
        return;
    }
    double gmax = cmax;
    gmax = fmax(gmax, __shfl_xor_sync(0xffffffffu, gmax, 1));
    gmax = fmax(gmax, __shfl_xor_sync(0xffffffffu, gmax, 2));
    int s = (int)clamp_rne(__dsub_rn(__ddiv_rn(__dmul_rn(4.0, gmax), __dmul_rn(43.0, d)), 0.5), 15.0);
    double db = __ddiv_rn(__dmul_rn(d, (double)(2 * s + 1)), 8.0);
    int neg[8], cnt = 0;
    for (int i = 0; i < 8; ++i) { neg[i] = xc[i] < 0.0f; cnt += neg[i]; }
    int flip = -1;
    if (cnt & 1) {
        double best = INFINITY;
        for (int i = 0; i < 8; ++i) {
            double a = fabs((double)xc[i]);
            if (a < best) { best = a; flip = i; }
        }
        neg[flip] = !neg[flip];
    }
    double t[8];
    for (int i = 0; i < 8; ++i) {
        double a = fabs((double)xc[i]);
        t[i] = (i == flip) ? -a : a;
    }
    int best_a = 0;
    double best_err = INFINITY;
    for (int a = 0; a < 256; ++a) {
        double err = 0.0;
        for (int i = 0; i < 8; ++i) {
            double diff = __dsub_rn(__dmul_rn(db, (double)sgrid[a * 8 + i]), t[i]);
            err = __dadd_rn(err, __dmul_rn(diff, diff));
        }
        if (err < best_err) { best_err = err; best_a = a; }
    }
    uint32_t sigma = 0;
    for (int i = 0; i < 7; ++i) sigma |= (uint32_t)neg[i] << i;
    int g = lane >> 2, c = lane & 3;
    uint32_t part = sigma << (7 * c);
    part |= __shfl_xor_sync(0xffffffffu, part, 1);
    part |= __shfl_xor_sync(0xffffffffu, part, 2);
    uint32_t S = part | ((uint32_t)s << 28);
    o[2 + 8 * g + c] = (uint8_t)best_a;
    if (c == 0) {
        o[2 + 8 * g + 4] = S & 0xff;
        o[2 + 8 * g + 5] = (S >> 8) & 0xff;
        o[2 + 8 * g + 6] = (S >> 16) & 0xff;
        o[2 + 8 * g + 7] = S >> 24;
    }
    if (lane == 0) { o[0] = dh & 0xff; o[1] = dh >> 8; }
}

// ---------------------------------------------------------------- repack
// IQ2 canonical blocks of an [R][C] matrix -> payload [R/32][C/64][32][16 B]
// (S words in the device order) and d [R/32][C/256][32].  One thread per (block, group).
__global__ void k_repack_iq2(const uint8_t* __restrict__ src, int R, int C, uint8_t* __restrict__ qs,
                             uint16_t* __restrict__ dd) {
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int64_t nb = (int64_t)R * C / kQK;
    if (gid >= nb * 8) return;
    int64_t b = gid >> 3;
    int g = (int)(gid & 7);
    int nsb = C / kQK;
    int r = (int)(b / nsb), sb = (int)(b % nsb);
    const uint8_t* blk = src + b * kIQ2Bytes;
    int kt = 4 * sb + (g >> 1), half = g & 1;
    uint8_t* dst = qs + (((int64_t)(r >> 5) * (C / 64) + kt) * 32 + (r & 31)) * 16 + half * 8;
    for (int i = 0; i < 4; ++i) dst[i] = blk[2 + 8 * g + i];
    const uint8_t* sp = blk + 2 + 8 * g + 4;
    const uint32_t S = iq2_s_to_device((uint32_t)sp[0] | ((uint32_t)sp[1] << 8) | ((uint32_t)sp[2] << 16) |
                                       ((uint32_t)sp[3] << 24));
    for (int i = 0; i < 4; ++i) dst[4 + i] = (uint8_t)(S >> (8 * i));
    if (g == 0) dd[((int64_t)(r >> 5) * nsb + sb) * 32 + (r & 31)] = (uint16_t)(blk[0] | (blk[1] << 8));
}

// Q2 canonical blocks of an [R][C] matrix (flat blocking) -> codes, scales,
// (d, dmin).  One thread per (row, 64-column step).
__global__ void k_repack_q2(const uint8_t* __restrict__ src, int R, int C, uint8_t* __restrict__ q,
                            uint32_t* __restrict__ sc, uint32_t* __restrict__ dd) {
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int nkt = C / 64;
    if (gid >= (int64_t)R * nkt) return;
    int r = (int)(gid / nkt), kt = (int)(gid % nkt);
    int64_t f0 = (int64_t)r * C + 64 * kt;
    const uint8_t* blk = src + (f0 / kQK) * kQ2Bytes;
    int o = (int)(f0 % kQK);
    int64_t piece = ((int64_t)(r >> 5) * nkt + kt) * 32 + (r & 31);
    uint8_t* qd = q + piece * 16;
    for (int i = 0; i < 16; ++i) qd[i] = blk[16 + o / 4 + i];
    sc[piece] = (uint32_t)blk[o / 16] | ((uint32_t)blk[o / 16 + 1] << 8) | ((uint32_t)blk[o / 16 + 2] << 16) |
                ((uint32_t)blk[o / 16 + 3] << 24);
    int nsb = C >= kQK ? C / kQK : 1;
    if ((64 * kt) % kQK == 0) {
        int sbi = (64 * kt) / kQK;
        if (sbi < nsb)
            dd[((int64_t)(r >> 5) * nsb + sbi) * 32 + (r & 31)] =
                (uint32_t)blk[80] | ((uint32_t)blk[81] << 8) | ((uint32_t)blk[82] << 16) | ((uint32_t)blk[83] << 24);
    }
}

// Q4 canonical blocks of an [R][C] matrix (C a multiple of 256) -> codes
// [R/32][C/64][32][32 B], scale words [R/32][C/64][32] and (d, dmin) words
// [R/32][C/256][32].  Code byte 8t + 4h + i/2 (nibble i & 1) of a row's
// 64-column step holds the code of column q4_dev_col(mode, t, h, i).  One
// thread per (row, 64-column step).
__global__ void k_repack_q4(const uint8_t* __restrict__ src, int R, int C, int mode, uint8_t* __restrict__ q,
                            uint32_t* __restrict__ sc, uint32_t* __restrict__ dd) {
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int nkt = C / 64;
    if (gid >= (int64_t)R * nkt) return;
    const int r = (int)(gid / nkt), kt = (int)(gid % nkt);
    const uint8_t* blk = src + ((int64_t)r * (C / kQK) + kt / 4) * kQ4Bytes;
    const int o = 64 * (kt % 4);   // first weight of the step in the block
    const int64_t piece = ((int64_t)(r >> 5) * nkt + kt) * 32 + (r & 31);
    uint8_t bytes[32];
    for (int i = 0; i < 32; ++i) bytes[i] = 0;
    for (int t = 0; t < 4; ++t)
        for (int h = 0; h < 2; ++h)
            for (int i = 0; i < 8; ++i) {
                const int c = o + q4_dev_col(mode, t, h, i);
                const uint32_t code = (blk[16 + c / 2] >> (4 * (c % 2))) & 15u;
                bytes[8 * t + 4 * h + i / 2] |= (uint8_t)(code << (4 * (i & 1)));
            }
    uint8_t* qd = q + piece * 32;
    for (int i = 0; i < 32; ++i) qd[i] = bytes[i];
    const int j0 = 2 * (kt % 4);   // the step's two 32-weight sub-blocks
    sc[piece] = (uint32_t)q4_field(blk, j0) | ((uint32_t)q4_field(blk, j0 + 1) << 8) |
                ((uint32_t)q4_field(blk, 8 + j0) << 16) | ((uint32_t)q4_field(blk, 9 + j0) << 24);
    if (kt % 4 == 0)
        dd[((int64_t)(r >> 5) * (C / kQK) + kt / 4) * 32 + (r & 31)] =
            (uint32_t)blk[0] | ((uint32_t)blk[1] << 8) | ((uint32_t)blk[2] << 16) | ((uint32_t)blk[3] << 24);
}

// bf16 row-major [R][C] -> core-matrix tiles [R/8][C/8][8][8].
__global__ void k_repack_bf16(const uint4* __restrict__ src, int R, int C, uint4* __restrict__ dst) {
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int nc8 = C / 8;
    if (gid >= (int64_t)R * nc8) return;
    int r = (int)(gid / nc8), c8 = (int)(gid % nc8);
    dst[((int64_t)(r >> 3) * nc8 + c8) * 8 + (r & 7)] = src[gid];
}

// Router rows [E][H] -> expert pairs interleaved per column [ceil(E/2)][H][2]
// (a missing partner of an odd last expert reads as zero).
__global__ void k_interleave_router(const float* __restrict__ W, int E, int H, float* __restrict__ W2) {
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t npairs = (E + 1) / 2;
    if (gid >= npairs * H) return;
    const int p = (int)(gid / H), c = (int)(gid % H);
    const int e0 = 2 * p, e1 = 2 * p + 1;
    W2[2 * gid] = W[(int64_t)e0 * H + c];
    W2[2 * gid + 1] = e1 < E ? W[(int64_t)e1 * H + c] : 0.f;
}

// Inverse views for the dequant hook: expert matrix -> row-major values.
__global__ void k_dequant_iq2(const uint8_t* __restrict__ qs, const uint16_t* __restrict__ dd,
                              const uint8_t* __restrict__ grid, int R, int C, float* out_f, __nv_bfloat16* out_b) {
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)R * C) return;
    int r = (int)(gid / C), col = (int)(gid % C);
    int kt = col / 64, within = col % 64;
    int half = within / 32, c = (within % 32) / 8, i = within % 8;
    const uint8_t* p = qs + (((int64_t)(r >> 5) * (C / 64) + kt) * 32 + (r & 31)) * 16 + half * 8;
    uint32_t S = (uint32_t)p[4] | ((uint32_t)p[5] << 8) | ((uint32_t)p[6] << 16) | ((uint32_t)p[7] << 24);
    float d = half_bits(dd[((int64_t)(r >> 5) * (C / kQK) + col / kQK) * 32 + (r & 31)]);
    float db = d * (float)(2 * iq2_dev_scale(S) + 1) * 0.125f;
    uint32_t sigma = iq2_dev_signs(S, c);
    uint32_t neg = i < 7 ? (sigma >> i) & 1u : (uint32_t)(__popc(sigma) & 1);
    float v = db * (float)grid[p[c] * 8 + i];
    v = neg ? -v : v;
    if (out_f) out_f[gid] = v;
    else out_b[gid] = __float2bfloat16_rn(v);
}

__global__ void k_dequant_q2(const uint8_t* __restrict__ q, const uint32_t* __restrict__ sc,
                             const uint32_t* __restrict__ dd, int R, int C, float* out_f, __nv_bfloat16* out_b) {
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)R * C) return;
    int r = (int)(gid / C), col = (int)(gid % C);
    int kt = col / 64, within = col % 64;
    int64_t piece = ((int64_t)(r >> 5) * (C / 64) + kt) * 32 + (r & 31);
    uint32_t code = (q[piece * 16 + within / 4] >> (2 * (within % 4))) & 3u;
    uint32_t sb = (sc[piece] >> (8 * (within / 16))) & 0xffu;
    int nsb = C >= kQK ? C / kQK : 1;
    uint32_t p = dd[((int64_t)(r >> 5) * nsb + (nsb > 1 ? col / kQK : 0)) * 32 + (r & 31)];
    float d = half_bits(p & 0xffffu), dmin = half_bits(p >> 16);
    float v = (d * (float)(sb & 15u)) * (float)code - dmin * (float)(sb >> 4);
    if (out_f) out_f[gid] = v;
    else out_b[gid] = __float2bfloat16_rn(v);
}

// One thread per (row, 64-column step): the step's 64 values.
__global__ void k_dequant_q4(const uint8_t* __restrict__ q, const uint32_t* __restrict__ sc,
                             const uint32_t* __restrict__ dd, int R, int C, int mode, float* out_f,
                             __nv_bfloat16* out_b) {
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int nkt = C / 64;
    if (gid >= (int64_t)R * nkt) return;
    const int r = (int)(gid / nkt), kt = (int)(gid % nkt);
    const int64_t piece = ((int64_t)(r >> 5) * nkt + kt) * 32 + (r & 31);
    const uint32_t sw = sc[piece];
    const uint32_t p = dd[((int64_t)(r >> 5) * (C / kQK) + kt / 4) * 32 + (r & 31)];
    const float d = half_bits(p & 0xffffu), dmin = half_bits(p >> 16);
    for (int t = 0; t < 4; ++t)
        for (int h = 0; h < 2; ++h)
            for (int i = 0; i < 8; ++i) {
                const int c = q4_dev_col(mode, t, h, i);
                const uint32_t code = (q[piece * 32 + 8 * t + 4 * h + i / 2] >> (4 * (i & 1))) & 15u;
                const int j = c / 32;
                const float v = (d * (float)((sw >> (8 * j)) & 0xffu)) * (float)code -
                                dmin * (float)((sw >> (16 + 8 * j)) & 0xffu);
                const int64_t at = (int64_t)r * C + 64 * kt + c;
                if (out_f) out_f[at] = v;
                else out_b[at] = __float2bfloat16_rn(v);
            }
}

__global__ void k_dequant_bf16_tiles(const __nv_bfloat16* __restrict__ t, int R, int C, float* out_f,
                                     __nv_bfloat16* out_b) {
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)R * C) return;
    int r = (int)(gid / C), col = (int)(gid % C);
    __nv_bfloat16 v = t[(((int64_t)(r >> 3) * (C / 8) + col / 8) * 8 + (r & 7)) * 8 + (col & 7)];
    if (out_f) out_f[gid] = __bfloat162float(v);
    else out_b[gid] = v;
}

}  // namespace ds4
