// decode.cu -- the fp32 GEMV plan for 1..decode_max tokens.
//
//   k_router_decode   logits in the canonical binary32 order, then (last CTA)
//                     top-k by (logit desc, index asc) and the softmax over
//                     the selected logits
//   k_gateup_decode   for every selected expert (each read once, applied to
//                     all tokens that chose it) and the shared expert:
//                     g = W_gate x, u = W_up x, h = silu(g) * u
//   k_down_decode     y = W_down h per selected expert slot and for the shared
//                     expert
//   k_combine_decode  out = y_shared + sum_j w_j y_j, j in rank order
//
// The weights are streamed once from HBM with 128-bit loads that skip L1;
// the IQ2 grid is expanded to binary32 in shared memory in 8 interleaved
// copies so that the per-lane random row lookups of a quarter warp never
// share a bank.  Work is split into row tasks handed out by an atomic queue,
// larger tasks first.
#include "ds4moe_internal.cuh"

namespace ds4 {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxSlots = 128;          // decode_max (<= 8) * top_k (<= 16)
constexpr int kTabFloats = 256 * 2 * 8 * 4;

// ---------------------------------------------------------------- router
__device__ __forceinline__ float4 load_x4(const void* x, int act_bf16, int64_t idx) {
    if (act_bf16) {
        uint2 v = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(x) + idx);
        return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                           __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
    }
    return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + idx);
}

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
    return v > bv || (v == bv && i < bi);
}

// Top-k and softmax of one token's logits by one warp.
__device__ void topk_softmax_warp(const float* logits, int E, int k, int32_t* ids, float* wts) {
    int lane = threadIdx.x & 31;
    uint32_t taken = 0;   // bit m: candidate lane + 32 m already chosen (E <= 1024)
    float my_l = 0.f;
    int my_id = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int m = 0; lane + 32 * m < E; ++m) {
            if (taken & (1u << m)) continue;
            int e = lane + 32 * m;
            float v = __ldcg(logits + e);
            if (better(v, e, bv, bi)) { bv = v; bi = e; }
        }
        for (int off = 16; off >= 1; off >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == j) { my_l = bv; my_id = bi; }
    }
    float lmax = __shfl_sync(0xffffffffu, my_l, 0);
    float ex = lane < k ? __expf(my_l - lmax) : 0.f;
    float den = ex;
    for (int off = 16; off >= 1; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    if (lane < k) {
        ids[lane] = my_id;
        wts[lane] = ex / den;
    }
}

template <int NT>
__global__ void __launch_bounds__(kThreads) k_router_decode(Weights W, Dims D, DecodeWs ws, const void* x, int n) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * kWarps + warp;
    const int H = D.H, E = D.E;
    if (e < E) {
        float acc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0.f;
        const float* wr = W.W_r + (int64_t)e * H + 4 * lane;
#pragma unroll 4
        for (int i = 0; i < H / 128; ++i) {
            float4 w4 = __ldg(reinterpret_cast<const float4*>(wr + 128 * i));
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (t < n) {
                    float4 x4 = load_x4(x, D.act_bf16, (int64_t)t * H + 128 * i + 4 * lane);
                    acc[t] = fmaf(x4.x, w4.x, acc[t]);
                    acc[t] = fmaf(x4.y, w4.y, acc[t]);
                    acc[t] = fmaf(x4.z, w4.z, acc[t]);
                    acc[t] = fmaf(x4.w, w4.w, acc[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) acc[t] = acc[t] + __shfl_xor_sync(0xffffffffu, acc[t], m);
        }
        if (lane == 0) {
            float b = W.b_r ? W.b_r[e] : 0.f;
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (t < n) ws.logits[(int64_t)t * E + e] = W.b_r ? acc[t] + b : acc[t];
        }
    }
    __shared__ bool s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        unsigned prev = atomicAdd(ws.ticket, 1u);
        s_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) {
        *ws.ticket = 0;
        *ws.queue1 = 0;
    }
    if (warp < n) topk_softmax_warp(ws.logits + (int64_t)warp * E, E, D.k, ws.ids + warp * D.k, ws.wts + warp * D.k);
}

// ---------------------------------------------------------------- routing table
// Unique selected experts in ascending order, and for each the slots
// (t * k + j) that chose it, in increasing slot order.
struct Routing {
    int nu;
    int uniq[kMaxSlots];
    int ustart[kMaxSlots + 1];
    int slot[kMaxSlots];
    int ids[kMaxSlots];
    int first[kMaxSlots];
};

__device__ void build_routing(Routing& R, const int32_t* ids, int nk) {
    int tid = threadIdx.x;
    if (tid < nk) R.ids[tid] = __ldcg(ids + tid);
    __syncthreads();
    int e = 0, pos = 0, first = 0;
    if (tid < nk) {
        e = R.ids[tid];
        first = 1;
        for (int s = 0; s < tid; ++s)
            if (R.ids[s] == e) { first = 0; ++pos; }
        R.first[tid] = first;
    }
    __syncthreads();
    int rank = 0;
    if (tid < nk) {
        for (int s = 0; s < nk; ++s)
            if (R.first[s] && R.ids[s] < e) ++rank;
    }
    if (tid < nk && first) {
        int cnt = 0;
        for (int s = 0; s < nk; ++s) cnt += R.ids[s] == e;
        R.uniq[rank] = e;
        R.ustart[rank + 1] = cnt;   // counts; prefix below
    }
    __syncthreads();
    if (tid == 0) {
        int nu = 0;
        for (int s = 0; s < nk; ++s) nu += R.first[s];
        R.nu = nu;
        R.ustart[0] = 0;
        for (int u = 0; u < nu; ++u) R.ustart[u + 1] += R.ustart[u];
    }
    __syncthreads();
    if (tid < nk) R.slot[R.ustart[rank] + pos] = tid;
    __syncthreads();
}

// ---------------------------------------------------------------- gate/up
// IQ2 group of 32 weights (4 chunks of 8) against NT token vectors.
template <int NT>
__device__ __forceinline__ void iq2_group(uint32_t idx, uint32_t S, float d, const float* __restrict__ tabp,
                                          const float* __restrict__ xcol, int H, const int* tok, int ns,
                                          float* acc) {
    float2 gs[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) gs[t] = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t a = (idx >> (8 * c)) & 255u;
        uint32_t sg = (S >> (7 * c)) & 127u;
        sg |= ((uint32_t)__popc(sg) & 1u) << 7;
        const float* trow = tabp + a * 64;
        float4 g0 = *reinterpret_cast<const float4*>(trow);
        float4 g1 = *reinterpret_cast<const float4*>(trow + 32);
        float w[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = __uint_as_float(__float_as_uint(w[i]) ^ ((sg << (31 - i)) & 0x80000000u));
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t < ns) {
                const float* xr = xcol + tok[t] * H + 8 * c;
                float4 x0 = *reinterpret_cast<const float4*>(xr);
                float4 x1 = *reinterpret_cast<const float4*>(xr + 4);
                gs[t] = ffma2(make_float2(w[0], w[1]), make_float2(x0.x, x0.y), gs[t]);
                gs[t] = ffma2(make_float2(w[2], w[3]), make_float2(x0.z, x0.w), gs[t]);
                gs[t] = ffma2(make_float2(w[4], w[5]), make_float2(x1.x, x1.y), gs[t]);
                gs[t] = ffma2(make_float2(w[6], w[7]), make_float2(x1.z, x1.w), gs[t]);
            }
        }
    }
    float db = d * (float)(2 * (S >> 28) + 1) * 0.125f;
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = fmaf(db, gs[t].x + gs[t].y, acc[t]);
}

// bf16x2 word -> two binary32 values, multiply-accumulated against x pairs.
__device__ __forceinline__ float2 bf16x2_fma(uint32_t wbits, float2 x, float2 acc) {
    return ffma2(make_float2(__uint_as_float(wbits << 16), __uint_as_float(wbits & 0xffff0000u)), x, acc);
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    k_gateup_decode(Weights W, Dims D, DecodeWs ws, const void* x, int n) {
    extern __shared__ __align__(16) float smem[];
    float* tab = smem;                      // kTabFloats
    float* xs = tab + kTabFloats;           // [n][H]
    float* red = xs + n * D.H;              // [kWarps][2][NT][32]
    __shared__ Routing R;
    __shared__ int s_task;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = D.H, I = D.I, k = D.k;
    if (blockIdx.x == 0 && tid == 0) *ws.queue2 = 0;

    for (int i = tid; i < kTabFloats; i += kThreads) {
        int a = i >> 6, hf = (i >> 5) & 1, j = i & 3;
        tab[i] = (float)W.grid_u8[a * 8 + hf * 4 + j];
    }
    for (int i = tid * 4; i < n * H; i += kThreads * 4) *reinterpret_cast<float4*>(xs + i) = load_x4(x, D.act_bf16, i);
    build_routing(R, ws.ids, n * k);   // syncs

    const int n_sh = D.has_shared ? I / 8 : 0;
    const int rb_per_e = I / 32;
    const int total = n_sh + R.nu * rb_per_e;
    const float* tabp = tab + (lane & 7) * 4;
    const int nkt = H / 64, nsb = H / 256;

    for (;;) {
        if (tid == 0) s_task = atomicAdd(ws.queue1, 1u);
        __syncthreads();
        const int task = s_task;
        if (task >= total) break;
        if (task < n_sh) {
            // shared expert rows 8*task .. +7; lane = (row, k-quarter)
            const int rr = lane & 7, kq = lane >> 3;
            const int64_t tile0 = (int64_t)task * (H / 8);
            float2 ag[NT], au[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) ag[t] = au[t] = make_float2(0.f, 0.f);
            constexpr int KB = 8;
            for (int kc0 = warp * 4 + kq; kc0 < H / 8; kc0 += 32 * KB) {
                uint4 wg[KB], wu[KB];
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    const int kc = kc0 + 32 * b;
                    if (kc < H / 8) {
                        wg[b] = ld_stream_v4(W.sh_gate + ((tile0 + kc) * 8 + rr) * 8);
                        wu[b] = ld_stream_v4(W.sh_up + ((tile0 + kc) * 8 + rr) * 8);
                    }
                }
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    const int kc = kc0 + 32 * b;
                    if (kc >= H / 8) break;
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        if (t < n) {
                            const float* xr = xs + t * H + 8 * kc;
                            float4 x0 = *reinterpret_cast<const float4*>(xr);
                            float4 x1 = *reinterpret_cast<const float4*>(xr + 4);
                            ag[t] = bf16x2_fma(wg[b].x, make_float2(x0.x, x0.y), ag[t]);
                            ag[t] = bf16x2_fma(wg[b].y, make_float2(x0.z, x0.w), ag[t]);
                            ag[t] = bf16x2_fma(wg[b].z, make_float2(x1.x, x1.y), ag[t]);
                            ag[t] = bf16x2_fma(wg[b].w, make_float2(x1.z, x1.w), ag[t]);
                            au[t] = bf16x2_fma(wu[b].x, make_float2(x0.x, x0.y), au[t]);
                            au[t] = bf16x2_fma(wu[b].y, make_float2(x0.z, x0.w), au[t]);
                            au[t] = bf16x2_fma(wu[b].z, make_float2(x1.x, x1.y), au[t]);
                            au[t] = bf16x2_fma(wu[b].w, make_float2(x1.z, x1.w), au[t]);
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                float g = ag[t].x + ag[t].y, u = au[t].x + au[t].y;
                g += __shfl_xor_sync(0xffffffffu, g, 8);
                g += __shfl_xor_sync(0xffffffffu, g, 16);
                u += __shfl_xor_sync(0xffffffffu, u, 8);
                u += __shfl_xor_sync(0xffffffffu, u, 16);
                if (kq == 0 && t < n) {
                    red[((warp * 2 + 0) * NT + t) * 32 + rr] = g;
                    red[((warp * 2 + 1) * NT + t) * 32 + rr] = u;
                }
            }
            __syncthreads();
            if (tid < 8 * n) {
                const int r = tid & 7, t = tid >> 3;
                float g = 0.f, u = 0.f;
                for (int w = 0; w < kWarps; ++w) {
                    g += red[((w * 2 + 0) * NT + t) * 32 + r];
                    u += red[((w * 2 + 1) * NT + t) * 32 + r];
                }
                ws.h_sh[(int64_t)t * I + 8 * task + r] = silu(g) * u;
            }
        } else {
            // routed expert uniq[u], rows 32*rb + lane
            const int tt = task - n_sh;
            const int u = tt / rb_per_e, rb = tt % rb_per_e;
            const int e = R.uniq[u];
            const int s0 = R.ustart[u], ns = R.ustart[u + 1] - s0;
            int tok[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) tok[t] = t < ns ? R.slot[s0 + t] / k : 0;
            float ag[NT], au[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) ag[t] = au[t] = 0.f;
            const uint8_t* gq = W.gate_qs + (int64_t)e * W.iq2_qs_stride + ((int64_t)rb * nkt * 32 + lane) * 16;
            const uint8_t* uq = W.up_qs + (int64_t)e * W.iq2_qs_stride + ((int64_t)rb * nkt * 32 + lane) * 16;
            const uint16_t* gd = W.gate_d + (int64_t)e * W.iq2_d_stride + (int64_t)rb * nsb * 32 + lane;
            const uint16_t* ud = W.up_d + (int64_t)e * W.iq2_d_stride + (int64_t)rb * nsb * 32 + lane;
            constexpr int KB = 8;
            for (int kt0 = warp * KB; kt0 < nkt; kt0 += kWarps * KB) {
                uint4 pg[KB], pu[KB];
                float dg[KB / 4], du[KB / 4];
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    if (kt0 + b < nkt) {
                        pg[b] = ld_stream_v4(gq + (int64_t)(kt0 + b) * 512);
                        pu[b] = ld_stream_v4(uq + (int64_t)(kt0 + b) * 512);
                    }
                }
#pragma unroll
                for (int b = 0; b < KB / 4; ++b) {
                    if (kt0 + 4 * b < nkt) {
                        dg[b] = half_bits(ld_stream_u16(gd + ((kt0 >> 2) + b) * 32));
                        du[b] = half_bits(ld_stream_u16(ud + ((kt0 >> 2) + b) * 32));
                    }
                }
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    const int kt = kt0 + b;
                    if (kt >= nkt) break;
                    const float* xcol = xs + 64 * kt;
                    iq2_group<NT>(pg[b].x, pg[b].y, dg[b >> 2], tabp, xcol, H, tok, ns, ag);
                    iq2_group<NT>(pg[b].z, pg[b].w, dg[b >> 2], tabp, xcol + 32, H, tok, ns, ag);
                    iq2_group<NT>(pu[b].x, pu[b].y, du[b >> 2], tabp, xcol, H, tok, ns, au);
                    iq2_group<NT>(pu[b].z, pu[b].w, du[b >> 2], tabp, xcol + 32, H, tok, ns, au);
                }
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (t < ns) {
                    red[((warp * 2 + 0) * NT + t) * 32 + lane] = ag[t];
                    red[((warp * 2 + 1) * NT + t) * 32 + lane] = au[t];
                }
            }
            __syncthreads();
            if (warp < ns) {
                const int t = warp;
                float g = 0.f, uu = 0.f;
                for (int w = 0; w < kWarps; ++w) {
                    g += red[((w * 2 + 0) * NT + t) * 32 + lane];
                    uu += red[((w * 2 + 1) * NT + t) * 32 + lane];
                }
                float h = silu(g) * uu;
                const int slot = R.slot[s0 + t];
                ws.h_rt[(int64_t)slot * I + 32 * rb + lane] = h;
                float hs = h;
#pragma unroll
                for (int m = 1; m <= 8; m <<= 1) hs += __shfl_xor_sync(0xffffffffu, hs, m);
                if ((lane & 15) == 0) ws.hsum_rt[(int64_t)slot * (I / 16) + 2 * rb + (lane >> 4)] = hs;
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- down
// sum_i (1 + q_i/4) h_i over the 16 codes of one 32-bit word, against NT slots.
template <int NT>
__device__ __forceinline__ void q2_word(uint32_t word, const float* const* hp, int ns, float* A) {
    uint32_t t0 = ((word << 5) & 0x60606060u) | 0x80808080u;
    uint32_t t1 = ((word << 3) & 0x60606060u) | 0x80808080u;
    uint32_t t2 = ((word << 1) & 0x60606060u) | 0x80808080u;
    uint32_t t3 = ((word >> 1) & 0x60606060u) | 0x80808080u;
    // byte j of t_k holds code 4j + k at bits 5..6 (over a set bit 7)
    float f[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t sel = 0x7044u | (uint32_t)(j << 8);
        f[4 * j + 0] = __uint_as_float(__byte_perm(t0, 0x3f000000u, sel));
        f[4 * j + 1] = __uint_as_float(__byte_perm(t1, 0x3f000000u, sel));
        f[4 * j + 2] = __uint_as_float(__byte_perm(t2, 0x3f000000u, sel));
        f[4 * j + 3] = __uint_as_float(__byte_perm(t3, 0x3f000000u, sel));
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if (t < ns) {
            float2 a = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
                float4 hv = *reinterpret_cast<const float4*>(hp[t] + i);
                a = ffma2(make_float2(f[i], f[i + 1]), make_float2(hv.x, hv.y), a);
                a = ffma2(make_float2(f[i + 2], f[i + 3]), make_float2(hv.z, hv.w), a);
            }
            A[t] = a.x + a.y;
        }
    }
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    k_down_decode(Weights W, Dims D, DecodeWs ws, int n) {
    extern __shared__ __align__(16) float smem[];
    float* hsh = smem;                      // [n][I] shared-expert h
    float* red = hsh + n * D.I;             // [kWarps][NT][32]
    __shared__ Routing R;
    __shared__ int s_task;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = D.H, I = D.I, k = D.k;

    if (D.has_shared)
        for (int i = tid * 4; i < n * I; i += kThreads * 4)
            *reinterpret_cast<float4*>(hsh + i) = __ldcg(reinterpret_cast<const float4*>(ws.h_sh + i));
    build_routing(R, ws.ids, n * k);

    const int n_sh = D.has_shared ? H / 8 : 0;
    const int rb_per_e = H / 32;
    const int total = n_sh + R.nu * rb_per_e;
    const int nkt = I / 64, nsb = I >= 256 ? I / 256 : 1;

    for (;;) {
        if (tid == 0) s_task = atomicAdd(ws.queue2, 1u);
        __syncthreads();
        const int task = s_task;
        if (task >= total) break;
        if (task < n_sh) {
            const int rr = lane & 7, kq = lane >> 3;
            const int64_t tile0 = (int64_t)task * (I / 8);
            float2 ay[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) ay[t] = make_float2(0.f, 0.f);
            constexpr int KB = 8;
            for (int kc0 = warp * 4 + kq; kc0 < I / 8; kc0 += 32 * KB) {
                uint4 wd[KB];
#pragma unroll
                for (int b = 0; b < KB; ++b)
                    if (kc0 + 32 * b < I / 8) wd[b] = ld_stream_v4(W.sh_down + ((tile0 + kc0 + 32 * b) * 8 + rr) * 8);
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    const int kc = kc0 + 32 * b;
                    if (kc >= I / 8) break;
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        if (t < n) {
                            const float* hr = hsh + t * I + 8 * kc;
                            float4 h0 = *reinterpret_cast<const float4*>(hr);
                            float4 h1 = *reinterpret_cast<const float4*>(hr + 4);
                            ay[t] = bf16x2_fma(wd[b].x, make_float2(h0.x, h0.y), ay[t]);
                            ay[t] = bf16x2_fma(wd[b].y, make_float2(h0.z, h0.w), ay[t]);
                            ay[t] = bf16x2_fma(wd[b].z, make_float2(h1.x, h1.y), ay[t]);
                            ay[t] = bf16x2_fma(wd[b].w, make_float2(h1.z, h1.w), ay[t]);
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                float y = ay[t].x + ay[t].y;
                y += __shfl_xor_sync(0xffffffffu, y, 8);
                y += __shfl_xor_sync(0xffffffffu, y, 16);
                if (kq == 0 && t < n) red[(warp * NT + t) * 32 + rr] = y;
            }
            __syncthreads();
            if (tid < 8 * n) {
                const int r = tid & 7, t = tid >> 3;
                float y = 0.f;
                for (int w = 0; w < kWarps; ++w) y += red[(w * NT + t) * 32 + r];
                ws.y_sh[(int64_t)t * H + 8 * task + r] = y;
            }
        } else {
            const int tt = task - n_sh;
            const int u = tt / rb_per_e, rb = tt % rb_per_e;
            const int e = R.uniq[u];
            const int s0 = R.ustart[u], ns = R.ustart[u + 1] - s0;
            int slot[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) slot[t] = t < ns ? R.slot[s0 + t] : 0;
            float acc[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[t] = 0.f;
            const uint8_t* qb = W.down_q + (int64_t)e * W.q2_q_stride + ((int64_t)rb * nkt * 32 + lane) * 16;
            const uint32_t* scb = W.down_sc + (int64_t)e * W.q2_sc_stride + (int64_t)rb * nkt * 32 + lane;
            const uint32_t* ddb = W.down_dd + (int64_t)e * W.q2_dd_stride + (int64_t)rb * nsb * 32 + lane;
            constexpr int KB = 4;
            for (int kt0 = warp * KB; kt0 < nkt; kt0 += kWarps * KB) {
                uint4 qv[KB];
                uint32_t scv[KB], ddv[KB];
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    const int kt = kt0 + b;
                    if (kt < nkt) {
                        qv[b] = ld_stream_v4(qb + (int64_t)kt * 512);
                        scv[b] = ld_stream_u32(scb + kt * 32);
                        ddv[b] = ld_stream_u32(ddb + (nsb > 1 ? (kt >> 2) : 0) * 32);
                    }
                }
#pragma unroll
                for (int b = 0; b < KB; ++b) {
                    const int kt = kt0 + b;
                    if (kt >= nkt) break;
                    const float d = half_bits(ddv[b] & 0xffffu), dmin = half_bits(ddv[b] >> 16);
                    const uint32_t words[4] = {qv[b].x, qv[b].y, qv[b].z, qv[b].w};
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const float* hp[NT];
                        float S[NT];
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            hp[t] = ws.h_rt + (int64_t)slot[t] * I + 64 * kt + 16 * jj;
                            S[t] = t < ns ? __ldg(ws.hsum_rt + (int64_t)slot[t] * (I / 16) + 4 * kt + jj) : 0.f;
                        }
                        float A[NT];
                        q2_word<NT>(words[jj], hp, ns, A);
                        const uint32_t sb = (scv[b] >> (8 * jj)) & 0xffu;
                        const float a4 = 4.0f * d * (float)(sb & 15u);
                        const float bb = a4 + dmin * (float)(sb >> 4);
#pragma unroll
                        for (int t = 0; t < NT; ++t)
                            if (t < ns) acc[t] = fmaf(a4, A[t], fmaf(-bb, S[t], acc[t]));
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (t < ns) red[(warp * NT + t) * 32 + lane] = acc[t];
            __syncthreads();
            if (warp < ns) {
                const int t = warp;
                float y = 0.f;
                for (int w = 0; w < kWarps; ++w) y += red[(w * NT + t) * 32 + lane];
                ws.y_rt[(int64_t)R.slot[s0 + t] * H + 32 * rb + lane] = y;
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- combine
__global__ void k_combine_decode(Dims D, DecodeWs ws, float* out, int n) {
    const int64_t i4 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    const int H = D.H, k = D.k;
    if (i4 >= (int64_t)n * H) return;
    const int t = (int)(i4 / H), r = (int)(i4 % H);
    float4 acc = D.has_shared ? __ldcg(reinterpret_cast<const float4*>(ws.y_sh + (int64_t)t * H + r))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const float w = __ldcg(ws.wts + t * k + j);
        const float4 y = __ldcg(reinterpret_cast<const float4*>(ws.y_rt + (int64_t)(t * k + j) * H + r));
        acc.x = fmaf(w, y.x, acc.x);
        acc.y = fmaf(w, y.y, acc.y);
        acc.z = fmaf(w, y.z, acc.z);
        acc.w = fmaf(w, y.w, acc.w);
    }
    *reinterpret_cast<float4*>(out + i4) = acc;
}

// ---------------------------------------------------------------- launchers
size_t gateup_smem_bytes(const Dims& D, int n, int NT) {
    return sizeof(float) * ((size_t)kTabFloats + (size_t)n * D.H + (size_t)kWarps * 2 * NT * 32);
}
size_t down_smem_bytes(const Dims& D, int n, int NT) {
    return sizeof(float) * ((size_t)n * D.I + (size_t)kWarps * NT * 32);
}

// Events (optional): ev[2i] / ev[2i+1] recorded around launch i.
struct Marks {
    cudaEvent_t const* ev;
    cudaStream_t st;
    int i = 0;
    void before() { if (ev) cudaEventRecord(ev[2 * i], st); }
    void after() { if (ev) cudaEventRecord(ev[2 * i + 1], st); ++i; }
};

const char* const kDecodeKernels[4] = {"k_router_decode", "k_gateup_decode", "k_down_decode", "k_combine_decode"};

// Per (kernel instance, device): dynamic shared memory opt-in and resident
// CTAs per SM, set once outside any stream capture.
struct KernelCfg {
    size_t smem = 0;
    int per_sm = 0;
};

template <typename K>
cudaError_t configure(K kernel, size_t smem, KernelCfg* cfg) {
    if (cfg->smem >= smem && cfg->per_sm > 0) return cudaSuccess;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    cfg->smem = smem;
    cfg->per_sm = per_sm;
    return cudaSuccess;
}

constexpr int kMaxDevices = 64;

template <int NT>
cudaError_t launch_decode_t(const Weights& W, const Dims& D, const DecodeWs& ws, const void* x, int n, float* out,
                            int n_sm, cudaStream_t st, cudaEvent_t const* ev) {
    static KernelCfg cfg1[kMaxDevices], cfg2[kMaxDevices];
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= kMaxDevices) return cudaErrorInvalidDevice;
    Marks mk{ev, st};
    const int rgrid = (D.E + kWarps - 1) / kWarps;
    const size_t s1 = gateup_smem_bytes(D, n, NT), s2 = down_smem_bytes(D, n, NT);
    if ((err = configure(k_gateup_decode<NT>, s1, &cfg1[dev])) != cudaSuccess) return err;
    if ((err = configure(k_down_decode<NT>, s2, &cfg2[dev])) != cudaSuccess) return err;
    mk.before();
    k_router_decode<NT><<<rgrid, kThreads, 0, st>>>(W, D, ws, x, n);
    mk.after();
    mk.before();
    k_gateup_decode<NT><<<n_sm * cfg1[dev].per_sm, kThreads, s1, st>>>(W, D, ws, x, n);
    mk.after();
    mk.before();
    k_down_decode<NT><<<n_sm * cfg2[dev].per_sm, kThreads, s2, st>>>(W, D, ws, n);
    mk.after();
    const int64_t n4 = (int64_t)n * D.H / 4;
    mk.before();
    k_combine_decode<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(D, ws, out, n);
    mk.after();
    return cudaGetLastError();
}

int decode_launches() { return 4; }
const char* decode_kernel_name(int i) { return (i >= 0 && i < 4) ? kDecodeKernels[i] : nullptr; }

cudaError_t launch_decode(const Weights& W, const Dims& D, const DecodeWs& ws, const void* x, int n, float* out,
                          int n_sm, cudaStream_t st, cudaEvent_t const* ev) {
    if (n <= 1) return launch_decode_t<1>(W, D, ws, x, n, out, n_sm, st, ev);
    if (n <= 2) return launch_decode_t<2>(W, D, ws, x, n, out, n_sm, st, ev);
    if (n <= 4) return launch_decode_t<4>(W, D, ws, x, n, out, n_sm, st, ev);
    return launch_decode_t<8>(W, D, ws, x, n, out, n_sm, st, ev);
}

cudaError_t launch_route(const Weights& W, const Dims& D, const DecodeWs& ws, const void* x, int n,
                         cudaStream_t st) {
    const int rgrid = (D.E + kWarps - 1) / kWarps;
    if (n <= 1) k_router_decode<1><<<rgrid, kThreads, 0, st>>>(W, D, ws, x, n);
    else if (n <= 2) k_router_decode<2><<<rgrid, kThreads, 0, st>>>(W, D, ws, x, n);
    else if (n <= 4) k_router_decode<4><<<rgrid, kThreads, 0, st>>>(W, D, ws, x, n);
    else k_router_decode<8><<<rgrid, kThreads, 0, st>>>(W, D, ws, x, n);
    return cudaGetLastError();
}

}  // namespace ds4
