// prefill.cu -- the bf16 tensor-core plan for more than decode_max tokens.
//
//   k_router_prefill   logits in the canonical binary32 order (each lane of a
//                      warp owns one of the 32 partial chains of a tile of
//                      8 tokens x 8 experts; butterfly at the end)
//   k_topk_prefill     warp per token: top-k and softmax over the selection
//   k_hist / k_scan / k_scatter   stable counting sort of the (token, slot)
//                      pairs by expert: slot s = t*k + j goes to position
//                      offs[e] + (number of earlier slots with the same expert)
//   k_gather           Xp[pos] = bf16(x[slot(pos) / k])
//   k_moe_gemm<mode>   persistent grouped GEMM on tcgen05: per (expert,
//                      256-row tile, n tile) D[256 x 256] = A[256 x K] B[256 x K]^T
//                      as two 128-row MMA halves sharing B; A = permuted
//                      activations (TMA, 128-byte swizzle), B = the expert's
//                      weights dequantized to bf16 in shared memory by eight
//                      warps (shared expert: copied by TMA), accumulators in
//                      TMEM, epilogue by eight warps: gate/up -> silu(g) * u
//                      as bf16, down -> binary32
//   k_combine_prefill  out = y_shared + sum_j w_j y_{pos(t, j)}, rank order
//                      (k_combine_steer_prefill: then y - F v (v . y))
#include <cuda.h>
#include <cudaTypedefs.h>

#include <map>
#include <mutex>
#include <utility>

#include "ds4moe_internal.cuh"
#include "tcgen05.cuh"
#include "topk.cuh"

namespace ds4 {

// ---------------------------------------------------------------- router
// CTA: 8 warps as 4 token groups x 2 expert groups, warp tile 8 tokens x 8
// experts (4 expert pairs) -> CTA tile 32 tokens x 16 experts.  The 32 x 128
// slices of x and of the pair-interleaved router rows (W_r2: for each column the
// weights of experts 2p and 2p+1 side by side) for each 128-column step stream
// into a kRP_S-stage shared-memory ring with 16-byte asynchronous copies (rows
// past n or E are zero-filled).  Lane L multiplies columns 4L .. 4L+3 of the
// slice into its chain, fma in column order; one packed FMA advances the
// chains of an expert pair, whose weights arrive as adjacent words.
constexpr int kRP_T = 32, kRP_E = 16, kRP_S = 4;
constexpr int kRP_Threads = 256;   // 8 warps; two CTAs per SM overlap each other's step barriers

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <bool BF16X>
__global__ void __launch_bounds__(kRP_Threads, 2) k_router_prefill(Weights W, Dims D, const void* x, int n, float* logits) {
    constexpr int XB = BF16X ? 2 : 4;                       // bytes per x element
    constexpr int XSTAGE = kRP_T * 128 * XB, WSTAGE = kRP_E * 128 * 4;
    extern __shared__ __align__(16) unsigned char rp_smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.x * kRP_T, e0 = blockIdx.y * kRP_E;
    const int wt = (warp & 3) * 8, wq = (warp >> 2) * 4;   // warp's 8 tokens / 4 expert pairs in the CTA tile
    const int H = D.H, E = D.E, steps = H / 128;
    const int npairs = (E + 1) / 2, p0 = e0 / 2;
    const unsigned char* xb = reinterpret_cast<const unsigned char*>(x);
    const unsigned char* w2 = reinterpret_cast<const unsigned char*>(W.W_r2);

    auto issue = [&](int i) {
        unsigned char* xs = rp_smem + (i % kRP_S) * (XSTAGE + WSTAGE);
        unsigned char* ws = xs + XSTAGE;
        // x: 32 rows x (128 * XB) bytes
        for (int q = tid; q < kRP_T * 8 * XB; q += kRP_Threads) {
            const int row = q / (8 * XB), c = q % (8 * XB);
            const int t = t0 + row;
            const bool ok = t < n;
            cp_async16(xs + row * 128 * XB + 16 * c, xb + ((int64_t)(ok ? t : 0) * H + 128 * i) * XB + 16 * c, ok);
        }
        // W_r2: kRP_E / 2 expert pairs x 1024 bytes
        for (int q = tid; q < (kRP_E / 2) * 64; q += kRP_Threads) {
            const int pr = q >> 6, c = q & 63;
            const int p = p0 + pr;
            const bool ok = p < npairs;
            // 16-byte chunk c holds columns 2c, 2c+1 of the pair; lane L reads chunks 2L and 2L+1,
            // stored 512 bytes apart so that each read of the warp is one contiguous 512-byte run
            cp_async16(ws + pr * 1024 + (c & 1) * 512 + (c >> 1) * 16,
                       w2 + ((int64_t)(ok ? p : 0) * H + 128 * i) * 8 + 16 * c, ok);
        }
    };

    float2 acc[8][4];   // [token][expert pair]
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kRP_S - 1; ++i) {
        if (i < steps) issue(i);
        cp_async_commit();
    }
    for (int i = 0; i < steps; ++i) {
        cp_async_wait<kRP_S - 2>();
        __syncthreads();   // step i has landed everywhere; step i-1's stage is free
        if (i + kRP_S - 1 < steps) issue(i + kRP_S - 1);
        cp_async_commit();
        const unsigned char* xs = rp_smem + (i % kRP_S) * (XSTAGE + WSTAGE);
        const float* ws = reinterpret_cast<const float*>(xs + XSTAGE);
        float4 wp[4][2];   // [pair][columns (0,1) | (2,3)] as (w_e, w_e+1) pairs
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            wp[b][0] = *reinterpret_cast<const float4*>(ws + (wq + b) * 256 + 4 * lane);
            wp[b][1] = *reinterpret_cast<const float4*>(ws + (wq + b) * 256 + 128 + 4 * lane);
        }
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            float4 xv;
            if (BF16X) {
                const uint2 v = *reinterpret_cast<const uint2*>(xs + ((wt + a) * 128 + 4 * lane) * 2);
                xv = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                                 __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
            } else {
                xv = *reinterpret_cast<const float4*>(xs + ((wt + a) * 128 + 4 * lane) * 4);
            }
            const float2 x0 = make_float2(xv.x, xv.x), x1 = make_float2(xv.y, xv.y);
            const float2 x2 = make_float2(xv.z, xv.z), x3 = make_float2(xv.w, xv.w);
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                acc[a][b] = ffma2(x0, make_float2(wp[b][0].x, wp[b][0].y), acc[a][b]);
                acc[a][b] = ffma2(x1, make_float2(wp[b][0].z, wp[b][0].w), acc[a][b]);
                acc[a][b] = ffma2(x2, make_float2(wp[b][1].x, wp[b][1].y), acc[a][b]);
                acc[a][b] = ffma2(x3, make_float2(wp[b][1].z, wp[b][1].w), acc[a][b]);
            }
        }
    }
    cp_async_wait<0>();
    // butterfly over the 32 chains, then one lane writes each logit
#pragma unroll
    for (int a = 0; a < 8; ++a) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            float lo = acc[a][b].x, hi = acc[a][b].y;
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) {
                lo = lo + __shfl_xor_sync(0xffffffffu, lo, m);
                hi = hi + __shfl_xor_sync(0xffffffffu, hi, m);
            }
            const int t = t0 + wt + a;
            const int e = e0 + 2 * (wq + b);
            if (lane == ((a * 4 + b) & 31) && t < n) {
                if (e < E) logits[(int64_t)t * E + e] = W.b_r ? lo + W.b_r[e] : lo;
                if (e + 1 < E) logits[(int64_t)t * E + e + 1] = W.b_r ? hi + W.b_r[e + 1] : hi;
            }
        }
    }
}

// Raises a kernel's dynamic shared-memory limit to at least `bytes`, once per
// (kernel, device) and thread-safe; the limit only ever grows.
static cudaError_t smem_opt_in(const void* kernel, int bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, int> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    int& cur = done[std::make_pair(kernel, dev)];
    if (cur >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) cur = bytes;
    return e;
}

// Launch of the router for n tokens (stage ring in dynamic shared memory).
static cudaError_t launch_router_prefill(const Weights& W, const Dims& D, const void* x, int n, float* logits,
                                         cudaStream_t st) {
    const dim3 grid((n + kRP_T - 1) / kRP_T, (D.E + kRP_E - 1) / kRP_E);
    cudaError_t e;
    if (D.act_bf16) {
        const int smem = kRP_S * (kRP_T * 128 * 2 + kRP_E * 128 * 4);
        if ((e = smem_opt_in(reinterpret_cast<const void*>(k_router_prefill<true>), smem)) != cudaSuccess) return e;
        k_router_prefill<true><<<grid, kRP_Threads, smem, st>>>(W, D, x, n, logits);
    } else {
        const int smem = kRP_S * (kRP_T * 128 * 4 + kRP_E * 128 * 4);
        if ((e = smem_opt_in(reinterpret_cast<const void*>(k_router_prefill<false>), smem)) != cudaSuccess) return e;
        k_router_prefill<false><<<grid, kRP_Threads, smem, st>>>(W, D, x, n, logits);
    }
    return cudaGetLastError();
}

__global__ void __launch_bounds__(256) k_topk_prefill(Dims D, const float* logits, int n, int32_t* ids, float* wts) {
    __shared__ float buf[8][1024];
    const int warp = threadIdx.x >> 5;
    const int t = blockIdx.x * 8 + warp;
    if (t >= n) return;
    topk_softmax_warp(logits + (int64_t)t * D.E, buf[warp], D.E, D.k, ids + (int64_t)t * D.k, wts + (int64_t)t * D.k);
}

// ---------------------------------------------------------------- grouped-GEMM tiling
// A tile is 256 rows (two 128-row tensor-core halves that share one dequantized
// B tile) by 256 columns, stepped 64 along K through three shared-memory stages.
constexpr int kGBM = 256, kGHalf = 128;
constexpr int kGBN = 256, kGBK = 64;
constexpr int kGStages = 3;
constexpr int kGAHalf = kGHalf * kGBK * 2;    // 16 KB
constexpr int kGAStage = 2 * kGAHalf;         // 32 KB
constexpr int kGBStage = kGBN * kGBK * 2;     // 32 KB
constexpr int kGDqWarps = 8, kGEpiWarps = 8;   // one dequantizing thread per B row
constexpr int kGWarps = 2 + kGDqWarps + kGEpiWarps;
constexpr int kGThreads = kGWarps * 32;
constexpr int kGSelRep = 16;                  // selector-table copies: conflict-free 8-byte reads
constexpr int kGSelBytes = 256 * kGSelRep * 8;
constexpr uint32_t kGTmemCols = 512;          // two 128-lane x 256-column binary32 accumulators

// ---------------------------------------------------------------- permutation
constexpr int kSortBlock = 1024;   // slots per block of the counting sort

__global__ void __launch_bounds__(kSortBlock) k_hist(const int32_t* ids, int nslots, int E, int32_t* blk_cnt) {
    extern __shared__ int cnt[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const int s = blockIdx.x * kSortBlock + threadIdx.x;
    if (s < nslots) atomicAdd(&cnt[ids[s]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) blk_cnt[(int64_t)blockIdx.x * E + e] = cnt[e];
}

// One CTA: counts, exclusive offsets, per-block offsets, and the m-tile prefix.
__global__ void __launch_bounds__(1024) k_scan(const int32_t* blk_cnt, int nblk, int E, int32_t* counts,
                                               int32_t* offs, int32_t* blk_off, int32_t* mt_prefix) {
    __shared__ int tot[1024], mt[1024];
    const int e = threadIdx.x;
    int c = 0;
    if (e < E)
        for (int b = 0; b < nblk; ++b) c += blk_cnt[(int64_t)b * E + e];
    tot[e] = e < E ? c : 0;
    mt[e] = e < E ? (c + kGBM - 1) / kGBM : 0;
    __syncthreads();
    if (e == 0) {
        int o = 0, m = 0;
        for (int q = 0; q < E; ++q) {
            const int cq = tot[q], mq = mt[q];
            offs[q] = o;
            mt_prefix[q] = m;
            o += cq;
            m += mq;
        }
        offs[E] = o;
        mt_prefix[E] = m;
    }
    __syncthreads();
    if (e < E) {
        counts[e] = c;
        int o = offs[e];
        for (int b = 0; b < nblk; ++b) {
            blk_off[(int64_t)b * E + e] = o;
            o += blk_cnt[(int64_t)b * E + e];
        }
    }
}

// Stable positions inside a block: rank among same-expert slots of the same
// warp (match_any), plus the counts of the block's earlier warps.
__global__ void __launch_bounds__(kSortBlock) k_scatter(const int32_t* ids, int nslots, int E, const int32_t* blk_off,
                                                        int32_t* pos_of_slot, int32_t* slot_of_pos) {
    extern __shared__ int wcnt[];   // [32 warps][E]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < 32 * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const int s = blockIdx.x * kSortBlock + tid;
    const int e = s < nslots ? ids[s] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && rank == 0) wcnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
        int before = 0;
        for (int w = 0; w < warp; ++w) before += wcnt[w * E + e];
        const int pos = blk_off[(int64_t)blockIdx.x * E + e] + before + rank;
        pos_of_slot[s] = pos;
        slot_of_pos[pos] = s;
    }
}

// Xp[pos][:] = bf16(x[slot / k][:]): 64 threads per row (4 rows per 256-thread
// block), 16-byte pieces, the row's source looked up once.
__global__ void __launch_bounds__(256) k_gather(const void* x, int act_bf16, const int32_t* slot_of_pos, int nslots,
                                                int k, int H, __nv_bfloat16* Xp) {
    const int pos = blockIdx.x * 4 + (threadIdx.x >> 6), l = threadIdx.x & 63;
    if (pos >= nslots) return;
    const int per = H / 8;
    const int64_t t = __ldg(slot_of_pos + pos) / k;
    uint4* dst = reinterpret_cast<uint4*>(Xp + (int64_t)pos * H);
    if (act_bf16) {
        const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(x) + t * H);
        for (int c8 = l; c8 < per; c8 += 64) dst[c8] = __ldg(src + c8);
    } else {
        const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + t * H);
        for (int c8 = l; c8 < per; c8 += 64) {
            const float4 a = __ldg(src + 2 * c8), b = __ldg(src + 2 * c8 + 1);
            dst[c8] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                                 pack_bf16x2(b.z, b.w));
        }
    }
}

// x (binary32) -> bf16, for the shared expert's A operand.
__global__ void k_to_bf16(const float* x, int64_t n8, __nv_bfloat16* xb) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n8) return;
    const float4 a = __ldg(reinterpret_cast<const float4*>(x) + 2 * g), b = __ldg(reinterpret_cast<const float4*>(x) + 2 * g + 1);
    reinterpret_cast<uint4*>(xb)[g] =
        make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
}

// ---------------------------------------------------------------- grouped GEMM
enum GemmMode : int { kModeGateUp = 0, kModeDown = 1, kModeShGateUp = 2, kModeShDown = 3 };

struct GemmArgs {
    Weights W;
    Dims D;
    const int32_t* counts;      // [E] rows per expert (routed modes)
    const int32_t* offs;        // [E + 1]
    const int32_t* mt_prefix;   // [E + 1] kGBM-row tiles per expert, prefix
    int n_rows;                 // shared modes: tokens
    __nv_bfloat16* out_h;       // gate/up modes: [rows][I] bf16
    float* out_y;               // down modes: [rows][H] binary32
    float* out_raw;             // gate/up modes, inspection only: when set, the binary32
                                // accumulators [rows][2I] (gate columns, then up) instead of h
    uint32_t* grid_refused;     // routed gate/up mode: set to 1 (grid has more than four magnitudes) or 0
    uint32_t* err;
};

struct GemmSmem {
    uint64_t fullA[kGStages], fullB[kGStages], empty[kGStages];
    uint64_t accF[2], accE[2], done;   // per accumulator buffer (TMEM columns 0..255, 256..511)
    uint32_t tmem_base;
    int abort;
    int nval;          // distinct grid magnitudes (gate/up mode)
    float gval[4];
};

__device__ __forceinline__ bool g_aborted(const GemmSmem& S) { return *(volatile const int*)&S.abort != 0; }
__device__ __forceinline__ void g_set_abort(GemmSmem& S) { *(volatile int*)&S.abort = 1; }

struct TileInfo {
    int e;        // expert (-1: shared)
    int row0;     // first row of the tile in A / the outputs
    int mvalid;   // rows of the tile that belong to the expert (1 .. kGBM)
    int nb;       // n tile
};

template <int MODE>
__device__ __forceinline__ TileInfo tile_info(const GemmArgs& a, int tile, int NB) {
    TileInfo ti;
    const int mtg = tile / NB;
    ti.nb = tile % NB;
    if (MODE == kModeGateUp || MODE == kModeDown) {
        int lo = 0, hi = a.D.E;   // largest e with mt_prefix[e] <= mtg
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldg(a.mt_prefix + mid) <= mtg) lo = mid;
            else hi = mid - 1;
        }
        const int mt = mtg - __ldg(a.mt_prefix + lo);
        ti.e = lo;
        ti.row0 = __ldg(a.offs + lo) + kGBM * mt;
        const int rem = __ldg(a.counts + lo) - kGBM * mt;
        ti.mvalid = rem < kGBM ? rem : kGBM;
    } else {
        ti.e = -1;
        ti.row0 = kGBM * mtg;
        const int rem = a.n_rows - ti.row0;
        ti.mvalid = rem < kGBM ? rem : kGBM;
    }
    return ti;
}

// B tiles are K-major core-matrix blocks (no swizzle): row r's 16-byte unit u
// (k = 8u .. 8u+7 of the 64-column step) sits at (r / 8) * 1024 + u * 128 +
// (r % 8) * 16, so eight consecutive rows fill one 128-byte line per unit.
__device__ __forceinline__ uint32_t b_row_off(int r) { return (uint32_t)((r >> 3) * 1024 + (r & 7) * 16); }

// IQ2 chunk (8 weights) -> 8 bf16 (16 bytes): d(2s+1)/8 * G[a][i] * (+-1).
// The grid holds at most four distinct magnitudes v_c, so each group of 32
// weights first rounds its four candidates d(2s+1)/8 * v_c to bf16 (the
// binary32 products are exact: at most 22 significant bits), held as bytes
// 0..7 of (cand01, cand23).  Row a of the selector table (sl, four 16-bit
// selectors loaded by the caller) gives, per pair of weights, the byte-permute
// selector that picks the two rounded candidates.  Rounding is symmetric, so
// the signs are applied to the picked pairs: sg * C_j places sign bit 2j at
// bit 15 and bit 2j+1 at bit 31 (the two shifted copies of the 8-bit sign byte
// do not overlap, so the multiply has no carries).
__device__ __forceinline__ uint4 iq2_chunk_bf16(uint2 sl, uint32_t S, int c, uint32_t cand01, uint32_t cand23) {
    const uint32_t sg = iq2_dev_signs(S, c);
    // sign of element 7 = parity of the seven stored bits, added at bit 31 of the last mask
    const uint32_t m3 = sg * 0x01000200u + ((uint32_t)__popc(sg) << 31);
    return make_uint4(__byte_perm(cand01, cand23, sl.x) ^ ((sg * 0x40008000u) & 0x80008000u),
                      __byte_perm(cand01, cand23, sl.x >> 16) ^ ((sg * 0x10002000u) & 0x80008000u),
                      __byte_perm(cand01, cand23, sl.y) ^ ((sg * 0x04000800u) & 0x80008000u),
                      __byte_perm(cand01, cand23, sl.y >> 16) ^ (m3 & 0x80008000u));
}

// Eight 2-bit codes (bits 2i of x, i = 0..7) -> 8 bf16 of (d sc) q - dmin m.
// Code i becomes the binary32 2^(23-2i) + q with one AND-OR (biased exponent
// 150 - 2i, the code left in place in the mantissa); subtracting 2^(23-2i) gives
// q exactly, and one FMA gives the binary32 weight before the bf16 rounding.
__device__ __forceinline__ uint4 q2_unit_bf16(uint32_t x, float2 sc2, float2 nmn2) {
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int i0 = 2 * j, i1 = 2 * j + 1;
        const float f0 = __uint_as_float(((150u - 2u * i0) << 23) | (x & (3u << (2 * i0))));
        const float f1 = __uint_as_float(((150u - 2u * i1) << 23) | (x & (3u << (2 * i1))));
        const float2 q = fadd2(make_float2(f0, f1), make_float2(-__uint_as_float((150u - 2u * i0) << 23),
                                                                -__uint_as_float((150u - 2u * i1) << 23)));
        const float2 w = ffma2(sc2, q, nmn2);
        o[j] = pack_bf16x2(w.x, w.y);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Eight 4-bit codes (byte j: column j in the low nibble, column 4 + j in the
// high nibble) -> 8 bf16 of (d sc) q - dmin m, columns 0..7.  With the two
// bytes of a pair in the low half of v, the nibble at bits b..b+3 (b <= 12,
// inside the mantissa) becomes the binary32 2^(23-b) + q with one AND-OR
// (biased exponent 150 - b), as in q2_unit_bf16; one FMA then rounds the
// weight once.
__device__ __forceinline__ uint4 q4_word_bf16(uint32_t x, float2 sc2, float2 nmn2) {
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // columns 2j, 2j+1: bytes 0, 1 (j even) or 2, 3 (j odd) of x; low nibbles for j < 2, high after
        const uint32_t v = (j & 1) ? (x >> 16) : (x & 0xffffu);
        const int b0 = (j & 2) ? 4 : 0, b1 = b0 + 8;
        const float f0 = __uint_as_float(((150u - b0) << 23) | (v & (15u << b0)));
        const float f1 = __uint_as_float(((150u - b1) << 23) | (v & (15u << b1)));
        const float2 q = fadd2(make_float2(f0, f1), make_float2(-__uint_as_float((150u - b0) << 23),
                                                                -__uint_as_float((150u - b1) << 23)));
        const float2 w = ffma2(sc2, q, nmn2);
        o[j] = pack_bf16x2(w.x, w.y);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// The eight codes of 16-byte unit 4h + p (columns 8(4h + p) .. +7 of a
// 64-column step) of a down row in the 4-bit code order (q4_dev_col mode 1:
// column 32h + 16 (p >> 1) + 8 (p & 1) + 4e + t sits at nibble p + 4e of word
// (t, h); wh[t] = word (t, h)), gathered into q4_word_bf16's byte order.
__device__ __forceinline__ uint32_t q4_down_unit(const uint32_t (&wh)[4], int p) {
    const uint32_t a0 = wh[0] >> (4 * p), a1 = wh[1] >> (4 * p), a2 = wh[2] >> (4 * p), a3 = wh[3] >> (4 * p);
    // nibble p of word t (e = 0) in the low nibble of byte t, nibble p + 4 (e = 1) in its high nibble
    const uint32_t lo = __byte_perm(__byte_perm(a0, a1, 0x0040u), __byte_perm(a2, a3, 0x0040u), 0x5410u);
    const uint32_t hi = __byte_perm(__byte_perm(a0, a1, 0x0062u), __byte_perm(a2, a3, 0x0062u), 0x5410u);
    return (lo & 0x0F0F0F0Fu) | ((hi & 0x0F0F0F0Fu) << 4);
}

// One dequantizing thread's packed weights for one k step (64 weights of one B row).
template <bool Q4>
struct BFrag {
    uint4 q;        // IQ2: two (grid indices, signs+scale) pairs; Q2: 64 codes; Q4: codes of columns 0..31
    uint32_t a0;    // IQ2: d (binary16 bits); Q2: four scale bytes; Q4: sc, sc, m, m of the two sub-blocks
    uint32_t a1;    // Q2, Q4: d | dmin << 16
};
template <>
struct BFrag<true> {
    uint4 q, q2;    // Q4: the row's 32 code bytes of the step
    uint32_t a0, a1;
};

// Warp roles: 0 TMA, 1 MMA, 2..9 dequantize B, 10..17 epilogue.  Q4: the routed
// experts are 4-bit blocks (no grid).
template <int MODE, bool Q4>
__global__ void __launch_bounds__(kGThreads, 1)
    k_moe_gemm(const __grid_constant__ CUtensorMap tmapA, const __grid_constant__ CUtensorMap tmapB0,
               const __grid_constant__ CUtensorMap tmapB1, GemmArgs a) {
    extern __shared__ __align__(1024) unsigned char g_smem_raw[];
    // 1024-byte aligned stages (the swizzle pattern repeats every 1024 bytes)
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(g_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char* stA = base;                                   // kGStages x 32 KB
    unsigned char* stB = base + kGStages * kGAStage;              // kGStages x 32 KB
    unsigned char* seltab = stB + kGStages * kGBStage;            // [256][kGSelRep] x 4 16-bit selectors
    __shared__ GemmSmem S;

    constexpr bool kRouted = MODE == kModeGateUp || MODE == kModeDown;
    constexpr bool kGateUp = MODE == kModeGateUp || MODE == kModeShGateUp;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.D.H, I = a.D.I;
    const int K = kGateUp ? H : I;
    const int KS = K / kGBK;
    const int NB = kGateUp ? I / 128 : H / kGBN;

    if (tid == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&S.fullA[s], 1);
            mbar_init(&S.fullB[s], kGDqWarps);
            mbar_init(&S.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&S.accF[b], 1);
            mbar_init(&S.accE[b], kGEpiWarps / 2);
        }
        mbar_init(&S.done, 1);
        S.abort = 0;
        fence_barrier_init();
    }
    if (MODE == kModeGateUp && Q4 && tid == 0 && blockIdx.x == 0 && a.grid_refused) *a.grid_refused = 0u;
    if (MODE == kModeGateUp && !Q4) {
        // magnitude classes of the grid bytes (stage A is free until the pipeline starts)
        int* present = reinterpret_cast<int*>(stA);
        int* cls = present + 256;
        for (int v = tid; v < 256; v += kGThreads) present[v] = 0;
        __syncthreads();
        for (int q = tid; q < 2048; q += kGThreads) present[a.W.grid_u8[q]] = 1;
        __syncthreads();
        if (tid == 0) {
            int nv = 0;
            for (int v = 0; v < 256; ++v) {
                cls[v] = nv < 4 ? nv : 3;
                if (present[v]) {
                    if (nv < 4) S.gval[nv] = (float)v;
                    ++nv;
                }
            }
            for (int c = nv; c < 4; ++c) S.gval[c] = 0.f;
            S.nval = nv;
            if (nv > 4) {
                set_err(a.err, kErrGrid);
                S.abort = 1;
            }
            if (blockIdx.x == 0 && a.grid_refused) *a.grid_refused = nv > 4 ? 1u : 0u;
        }
        __syncthreads();
        for (int row = tid; row < 256; row += kGThreads) {
            uint32_t sel[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t ca = (uint32_t)cls[a.W.grid_u8[row * 8 + 2 * j]];
                const uint32_t cb = (uint32_t)cls[a.W.grid_u8[row * 8 + 2 * j + 1]];
                sel[j] = 0x1010u + 0x22u * ca + 0x2200u * cb;   // bytes 2c, 2c+1 hold candidate c
            }
            const uint2 ent = make_uint2(sel[0] | (sel[1] << 16), sel[2] | (sel[3] << 16));
#pragma unroll
            for (int p = 0; p < kGSelRep; ++p)
                *reinterpret_cast<uint2*>(seltab + row * (kGSelRep * 8) + p * 8) = ent;
        }
    }
    if (warp == 1) {
        tmem_alloc(&S.tmem_base, kGTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const int total_mt = kRouted ? __ldg(a.mt_prefix + a.D.E) : (a.n_rows + kGBM - 1) / kGBM;
    const int ntiles = total_mt * NB;

    if (warp == 0) {
        // ------------------------------------------------ A tiles (and shared-expert B tiles) by TMA
        uint32_t it = 0;
        for (int tile = blockIdx.x; tile < ntiles && !g_aborted(S); tile += gridDim.x) {
            const TileInfo ti = tile_info<MODE>(a, tile, NB);
            const bool two = ti.mvalid > kGHalf;
            for (int ks = 0; ks < KS; ++ks, ++it) {
                const int s = it % kGStages;
                if (!mbar_wait(&S.empty[s], ((it / kGStages) & 1) ^ 1, a.err)) { g_set_abort(S); break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&S.fullA[s], (two ? 2 : 1) * kGAHalf + (kRouted ? 0 : kGBStage));
                    tma_load_2d(stA + s * kGAStage, &tmapA, ks * kGBK, ti.row0, &S.fullA[s]);
                    if (two) tma_load_2d(stA + s * kGAStage + kGAHalf, &tmapA, ks * kGBK, ti.row0 + kGHalf, &S.fullA[s]);
                    if (MODE == kModeShGateUp) {   // rows 0..127: gate rows, 128..255: up rows of n tile nb
                        tma_load_3d(stB + s * kGBStage, &tmapB0, 0, 8 * ks, 16 * ti.nb, &S.fullA[s]);
                        tma_load_3d(stB + s * kGBStage + kGBStage / 2, &tmapB1, 0, 8 * ks, 16 * ti.nb, &S.fullA[s]);
                    } else if (MODE == kModeShDown) {
                        tma_load_3d(stB + s * kGBStage, &tmapB0, 0, 8 * ks, 32 * ti.nb, &S.fullA[s]);
                        tma_load_3d(stB + s * kGBStage + kGBStage / 2, &tmapB0, 0, 8 * ks, 32 * ti.nb + 16,
                                    &S.fullA[s]);
                    }
                }
                __syncwarp();
            }
        }
        // drain: the last issued copies land before the CTA leaves
        const uint32_t j0 = it > (uint32_t)kGStages ? it - kGStages : 0;
        for (uint32_t j = j0; j < it; ++j) mbar_wait(&S.fullA[j % kGStages], (j / kGStages) & 1, a.err);
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issue: two 128 x 256 x 16 MMAs per k16 share B
        const uint32_t idesc = umma_idesc_bf16(kGHalf, kGBN);
        // A 256-row tile uses both accumulator buffers (its two row halves); a tile of at most 128
        // rows uses one, alternating, so that its epilogue overlaps the next such tile's MMAs.
        uint32_t it = 0, use0 = 0, use1 = 0, hc = 0;   // completed uses of each buffer
        for (int tile = blockIdx.x; tile < ntiles && !g_aborted(S); tile += gridDim.x) {
            const TileInfo ti = tile_info<MODE>(a, tile, NB);
            const bool two = ti.mvalid > kGHalf;
            const int b1 = two ? 0 : (int)(hc++ & 1u);   // buffer of the tile's first row half
            if (!mbar_wait(&S.accE[b1], ((b1 ? use1 : use0) & 1) ^ 1, a.err) ||
                (two && !mbar_wait(&S.accE[1], (use1 & 1) ^ 1, a.err))) {
                g_set_abort(S);
                break;
            }
            tc_fence_after();
            const uint32_t dt0 = tmem + (uint32_t)b1 * kGBN;
            for (int ks = 0; ks < KS; ++ks, ++it) {
                const int s = it % kGStages;
                const uint32_t ph = (it / kGStages) & 1;
                if (!mbar_wait(&S.fullA[s], ph, a.err) || (kRouted && !mbar_wait(&S.fullB[s], ph, a.err))) {
                    g_set_abort(S);
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t da0 = umma_desc_sw128(smem_addr(stA + s * kGAStage));
                    const uint64_t da1 = umma_desc_sw128(smem_addr(stA + s * kGAStage + kGAHalf));
                    // B (dequantized or copied) is in core-matrix blocks: K advance per 16 elements is
                    // two 128-byte blocks; A is 128-byte swizzled: 32 bytes per 16 elements
                    const uint64_t db = umma_desc_core(smem_addr(stB + s * kGBStage));
                    constexpr uint32_t bstep = 16u;
#pragma unroll
                    for (int kk = 0; kk < kGBK / 16; ++kk) {
                        umma_bf16(dt0, da0 + 2 * kk, db + bstep * kk, idesc, (ks | kk) != 0);
                        if (two) umma_bf16(tmem + kGBN, da1 + 2 * kk, db + bstep * kk, idesc, (ks | kk) != 0);
                    }
                    umma_commit(&S.empty[s]);
                }
                __syncwarp();
            }
            if (g_aborted(S)) break;
            if (lane == 0) {
                umma_commit(&S.accF[b1]);
                if (two) umma_commit(&S.accF[1]);
            }
            __syncwarp();
            if (two || b1 == 0) ++use0;
            if (two || b1 == 1) ++use1;
        }
        // every issued MMA has finished before TMEM is released
        if (lane == 0) umma_commit(&S.done);
        __syncwarp();
        mbar_wait(&S.done, 0, a.err);
    } else if (warp < 2 + kGDqWarps) {
        // ------------------------------------------------ B tiles (dequantize to bf16)
        if (kRouted) {
            const int r = tid - 64;   // B-tile row 0..255
            const unsigned char* selp = seltab + (lane & 15) * 8;
            float2 gv01 = make_float2(0.f, 0.f), gv23 = make_float2(0.f, 0.f);
            if (MODE == kModeGateUp && !Q4) {
                gv01 = make_float2(S.gval[0], S.gval[1]);
                gv23 = make_float2(S.gval[2], S.gval[3]);
            }
            const int my_tiles = (int)blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
            const int total = my_tiles * KS;
            // load cursor: tile, k step and this row's packed-weight pointers
            int ctile = blockIdx.x, cks = 0;
            const uint8_t* qs = nullptr;
            const uint16_t* dq = nullptr;
            const uint32_t* scp = nullptr;
            const uint32_t* ddp = nullptr;
            // an expert with more than one row tile has its weights read by each of them (its row tiles
            // run on neighbouring CTAs at about the same time): keep those weights in L2
            const uint64_t pol_keep = policy_evict_last();
            bool keep = false;
            auto set_src = [&](int tile) {
                const TileInfo ti = tile_info<MODE>(a, tile, NB);
                const size_t e = (size_t)ti.e;
                keep = __ldg(a.counts + e) > kGBM;
                if (Q4) {
                    // codes [R/32][C/64][32][32 B], scale words [R/32][C/64][32], (d, dmin) [R/32][C/256][32]
                    const bool gu = MODE == kModeGateUp;
                    const int row = gu ? 128 * ti.nb + (r & 127) : kGBN * ti.nb + r;
                    const int nkt = (gu ? H : I) / 64, nsb = (gu ? H : I) / 256;
                    const uint8_t* qb = gu ? (r < 128 ? a.W.gate_qs : a.W.up_qs) : a.W.down_q;
                    const uint32_t* sb = gu ? (r < 128 ? a.W.gate_sc4 : a.W.up_sc4) : a.W.down_sc4;
                    const uint32_t* db = gu ? (r < 128 ? a.W.gate_dd4 : a.W.up_dd4) : a.W.down_dd4;
                    qs = qb + e * a.W.q4_q_stride + ((size_t)(row >> 5) * nkt * 32 + (row & 31)) * 32;
                    scp = sb + e * a.W.q4_sc_stride + (size_t)(row >> 5) * nkt * 32 + (row & 31);
                    ddp = db + e * a.W.q4_dd_stride + (size_t)(row >> 5) * nsb * 32 + (row & 31);
                } else if (MODE == kModeGateUp) {
                    const int row = 128 * ti.nb + (r & 127);
                    qs = (r < 128 ? a.W.gate_qs : a.W.up_qs) + e * a.W.iq2_qs_stride +
                         (size_t)(row >> 5) * (H / 64) * 512 + (row & 31) * 16;
                    dq = (r < 128 ? a.W.gate_d : a.W.up_d) + e * a.W.iq2_d_stride + (size_t)(row >> 5) * (H / 256) * 32 +
                         (row & 31);
                } else {
                    const int row = kGBN * ti.nb + r;
                    const int nkt = I / 64, nsb = I >= 256 ? I / 256 : 1;
                    qs = a.W.down_q + e * a.W.q2_q_stride + ((size_t)(row >> 5) * nkt * 32 + (row & 31)) * 16;
                    scp = a.W.down_sc + e * a.W.q2_sc_stride + (size_t)(row >> 5) * nkt * 32 + (row & 31);
                    ddp = a.W.down_dd + e * a.W.q2_dd_stride + (size_t)(row >> 5) * nsb * 32 + (row & 31);
                }
            };
            auto fetch = [&](BFrag<Q4>& f) {
                if constexpr (Q4) {
                    const uint8_t* src = qs + (size_t)cks * 1024;
                    f.q = keep ? ld_stream_v4_hint(src, pol_keep) : ld_stream_v4(src);
                    f.q2 = keep ? ld_stream_v4_hint(src + 16, pol_keep) : ld_stream_v4(src + 16);
                    f.a0 = ld_stream_u32(scp + cks * 32);
                    f.a1 = ld_stream_u32(ddp + (cks >> 2) * 32);
                } else {
                f.q = keep ? ld_stream_v4_hint(qs + (size_t)cks * 512, pol_keep) : ld_stream_v4(qs + (size_t)cks * 512);
                if (MODE == kModeGateUp) {
                    f.a0 = ld_stream_u16(dq + (cks >> 2) * 32);
                } else {
                    f.a0 = ld_stream_u32(scp + cks * 32);
                    f.a1 = ld_stream_u32(ddp + (I >= 256 ? (cks >> 2) : 0) * 32);
                }
                }
                if (++cks == KS) {
                    cks = 0;
                    ctile += gridDim.x;
                    if (ctile < ntiles) set_src(ctile);
                }
            };
            constexpr int PD = Q4 ? 2 : 4;   // k steps of packed weights in flight (4-bit steps are 32 bytes)
            BFrag<Q4> ring[PD];
            if (total > 0) set_src(ctile);
#pragma unroll
            for (int p = 0; p < PD; ++p)
                if (p < total) fetch(ring[p]);
            uint32_t it = 0;
            for (int j0 = 0; j0 < total && !g_aborted(S); j0 += PD) {
#pragma unroll
                for (int p = 0; p < PD; ++p) {
                    if (j0 + p >= total) break;
                    const BFrag<Q4> cur = ring[p];
                    if (j0 + p + PD < total) fetch(ring[p]);
                    const int s = it % kGStages;
                    if (!mbar_wait(&S.empty[s], ((it / kGStages) & 1) ^ 1, a.err)) {
                        g_set_abort(S);
                        break;
                    }
                    unsigned char* bt = stB + s * kGBStage + b_row_off(r);
                    if constexpr (Q4) {
                        // 16-byte unit c = columns 8c .. 8c+7, in the 32-column sub-block c >> 2
                        const float d = half_bits(cur.a1 & 0xffffu), dmin = half_bits(cur.a1 >> 16);
                        // one 32-column half at a time (both unrolled spill at the 96-register budget); word
                        // (t, h) of the step is code bytes 8t + 4h .. +3
#pragma unroll 1
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t wh[4] = {h ? cur.q.y : cur.q.x, h ? cur.q.w : cur.q.z,
                                                    h ? cur.q2.y : cur.q2.x, h ? cur.q2.w : cur.q2.z};
                            const float sc = d * (float)((cur.a0 >> (8 * h)) & 0xffu);
                            const float mn = dmin * (float)((cur.a0 >> (16 + 8 * h)) & 0xffu);
                            const float2 sc2 = make_float2(sc, sc), nmn2 = make_float2(-mn, -mn);
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                // gate/up (code order mode 0): unit 4h + t is word (t, h) as it stands
                                const uint32_t x = MODE == kModeGateUp ? wh[t] : q4_down_unit(wh, t);
                                *reinterpret_cast<uint4*>(bt + (4 * h + t) * 128) = q4_word_bf16(x, sc2, nmn2);
                            }
                        }
                    } else if (MODE == kModeGateUp) {
                        const float d = half_bits(cur.a0);
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            // the group's four selector rows first: the loads then overlap instead of
                            // waiting behind the tile stores (which the compiler cannot reorder)
                            const uint32_t idx = hf ? cur.q.z : cur.q.x, Sw = hf ? cur.q.w : cur.q.y;
                            uint2 sl[4];
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                sl[c] = *reinterpret_cast<const uint2*>(selp + __byte_perm(idx, 0u, 0x4440u | c) *
                                                                                   (kGSelRep * 8));
                            const float db =
                                d * (__uint_as_float(0x4b000001u | (iq2_dev_scale(Sw) << 1)) - 8388608.0f) * 0.125f;
                            const float2 db2 = make_float2(db, db);
                            const float2 c01 = fmul2(db2, gv01), c23 = fmul2(db2, gv23);
                            const uint32_t cand01 = pack_bf16x2(c01.x, c01.y), cand23 = pack_bf16x2(c23.x, c23.y);
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                *reinterpret_cast<uint4*>(bt + (4 * hf + c) * 128) =
                                    iq2_chunk_bf16(sl[c], Sw, c, cand01, cand23);
                        }
                    } else {
                        const float d = half_bits(cur.a1 & 0xffffu), dmin = half_bits(cur.a1 >> 16);
                        // two sub-blocks per pass: a full unroll schedules all eight units at once and spills
#pragma unroll 2
                        for (int sbk = 0; sbk < 4; ++sbk) {
                            const uint32_t w = (sbk & 2) ? ((sbk & 1) ? cur.q.w : cur.q.z) : ((sbk & 1) ? cur.q.y : cur.q.x);
                            const uint32_t sb = (cur.a0 >> (8 * sbk)) & 0xffu;
                            const float sc = d * (float)(sb & 15u), mn = dmin * (float)(sb >> 4);
                            const float2 sc2 = make_float2(sc, sc), nmn2 = make_float2(-mn, -mn);
                            *reinterpret_cast<uint4*>(bt + (2 * sbk) * 128) = q2_unit_bf16(w, sc2, nmn2);
                            *reinterpret_cast<uint4*>(bt + (2 * sbk + 1) * 128) = q2_unit_bf16(w >> 16, sc2, nmn2);
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.fullB[s]);
                    ++it;
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue (TMEM -> registers -> global)
        // warps 10..13 drain buffer 0 and warps 14..17 buffer 1, following the MMA warp's assignment
        const int qd = warp & 3;                          // TMEM lanes 32 qd .. 32 qd + 31
        const int bg = (warp - 2 - kGDqWarps) >> 2;       // accumulator buffer of this warp
        uint32_t use = 0, hc = 0;
        for (int tile = blockIdx.x; tile < ntiles && !g_aborted(S); tile += gridDim.x) {
            const TileInfo ti = tile_info<MODE>(a, tile, NB);
            const bool two = ti.mvalid > kGHalf;
            const int b1 = two ? 0 : (int)(hc++ & 1u);
            if (!two && b1 != bg) continue;               // the other buffer's warps drain this tile
            const int half = two ? bg : 0;                // row half of the tile held in this buffer
            const int m = kGHalf * half + 32 * qd + lane; // tile row of this thread
            if (!mbar_wait(&S.accF[bg], use & 1, a.err)) { g_set_abort(S); break; }
            ++use;
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(32 * qd) << 16) + bg * kGBN;
            const bool live = m < ti.mvalid;
            {
                // 16-column TMEM reads; each thread stores 32-byte pieces of its own row
                if (kGateUp && a.out_raw) {
                    // inspection: the accumulators as they are (no SwiGLU)
                    float* dg = a.out_raw + (size_t)(ti.row0 + m) * 2 * I + 128 * ti.nb;
#pragma unroll 1
                    for (int c0 = 0; c0 < 128; c0 += 16) {
                        uint32_t g[16], u[16];
                        tmem_ld_32x16(taddr + c0, g);
                        tmem_ld_32x16(taddr + 128 + c0, u);
                        tmem_wait_ld();
                        if (live) {
                            st_global_v8(dg + c0, g[0], g[1], g[2], g[3], g[4], g[5], g[6], g[7]);
                            st_global_v8(dg + c0 + 8, g[8], g[9], g[10], g[11], g[12], g[13], g[14], g[15]);
                            st_global_v8(dg + I + c0, u[0], u[1], u[2], u[3], u[4], u[5], u[6], u[7]);
                            st_global_v8(dg + I + c0 + 8, u[8], u[9], u[10], u[11], u[12], u[13], u[14], u[15]);
                        }
                    }
                } else if (kGateUp) {
                    __nv_bfloat16* dst = a.out_h + (size_t)(ti.row0 + m) * I + 128 * ti.nb;
#pragma unroll 1
                    for (int c0 = 0; c0 < 128; c0 += 16) {
                        uint32_t g[16], u[16];
                        tmem_ld_32x16(taddr + c0, g);
                        tmem_ld_32x16(taddr + 128 + c0, u);
                        tmem_wait_ld();
                        uint32_t hp[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float h0 = silu(__uint_as_float(g[2 * j])) * __uint_as_float(u[2 * j]);
                            const float h1 = silu(__uint_as_float(g[2 * j + 1])) * __uint_as_float(u[2 * j + 1]);
                            hp[j] = pack_bf16x2(h0, h1);
                        }
                        if (live) st_global_v8(dst + c0, hp[0], hp[1], hp[2], hp[3], hp[4], hp[5], hp[6], hp[7]);
                    }
                } else {
                    float* dst = a.out_y + (size_t)(ti.row0 + m) * H + kGBN * ti.nb;
#pragma unroll 1
                    for (int c0 = 0; c0 < kGBN; c0 += 16) {
                        uint32_t v[16];
                        tmem_ld_32x16(taddr + c0, v);
                        tmem_wait_ld();
                        if (live) {
                            st_global_v8(dst + c0, v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
                            st_global_v8(dst + c0 + 8, v[8], v[9], v[10], v[11], v[12], v[13], v[14], v[15]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.accE[bg]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kGTmemCols);
    }
}

// ---------------------------------------------------------------- combine
__global__ void k_combine_prefill(Dims D, const float* ys, const float* y, const float* wts, const int32_t* pos_of_slot,
                                  int n, const void* xres, const uint32_t* grid_refused, float* out) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // float4 index
    const int H = D.H, k = D.k;
    if (g >= (int64_t)n * H / 4) return;
    if (__ldcg(grid_refused)) return;   // this call's routed GEMMs refused the grid: out stays as it was
    const int t = (int)(g / (H / 4)), r4 = (int)(g % (H / 4));
    float4 acc = D.has_shared ? __ldg(reinterpret_cast<const float4*>(ys + (int64_t)t * H) + r4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const float w = __ldg(wts + (int64_t)t * k + j);
        const int pos = __ldg(pos_of_slot + (int64_t)t * k + j);
        const float4 v = __ldg(reinterpret_cast<const float4*>(y + (int64_t)pos * H) + r4);
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
    }
    if (xres) {   // out = x + layer(x)
        const int64_t e0 = (int64_t)t * H + 4 * r4;
        acc = make_float4(act_at(xres, e0, D.act_bf16) + acc.x, act_at(xres, e0 + 1, D.act_bf16) + acc.y,
                          act_at(xres, e0 + 2, D.act_bf16) + acc.z, act_at(xres, e0 + 3, D.act_bf16) + acc.w);
    }
    reinterpret_cast<float4*>(out + (int64_t)t * H)[r4] = acc;
}

// The combine with directional steering of the layer output (one CTA per
// token): y as above, then y - F v (v . y) with v . y summed in a fixed order,
// then x + that when the call asks for the residual.
constexpr int kSteerThreadsP = 256;

__global__ void __launch_bounds__(kSteerThreadsP) k_combine_steer_prefill(Dims D, const float* ys, const float* y,
                                                                          const float* wts, const int32_t* pos_of_slot,
                                                                          const float* v, float F, const void* xres,
                                                                          const uint32_t* grid_refused, float* out) {
    __shared__ float red[kSteerThreadsP / 32];
    if (__ldcg(grid_refused)) return;   // this call's routed GEMMs refused the grid: out stays as it was
    __shared__ int s_pos[16];
    __shared__ float s_w[16];
    const int t = blockIdx.x, H = D.H, k = D.k;
    if (threadIdx.x < k) {
        s_pos[threadIdx.x] = __ldg(pos_of_slot + (int64_t)t * k + threadIdx.x);
        s_w[threadIdx.x] = __ldg(wts + (int64_t)t * k + threadIdx.x);
    }
    __syncthreads();
    float4 acc[4];   // H <= 4096: four float4 column groups per thread
    float dot = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int c4 = threadIdx.x + q * kSteerThreadsP;   // float4 index in the row
        if (4 * c4 < H) {
            float4 a = D.has_shared ? __ldg(reinterpret_cast<const float4*>(ys + (int64_t)t * H) + c4)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < k; ++j) {
                const float w = s_w[j];
                const float4 yv = __ldg(reinterpret_cast<const float4*>(y + (int64_t)s_pos[j] * H) + c4);
                a.x = fmaf(w, yv.x, a.x);
                a.y = fmaf(w, yv.y, a.y);
                a.z = fmaf(w, yv.z, a.z);
                a.w = fmaf(w, yv.w, a.w);
            }
            acc[q] = a;
            const float4 vv = __ldg(reinterpret_cast<const float4*>(v) + c4);
            dot = fmaf(vv.x, a.x, dot);
            dot = fmaf(vv.y, a.y, dot);
            dot = fmaf(vv.z, a.z, dot);
            dot = fmaf(vv.w, a.w, dot);
        }
    }
    const float sF = F * cta_sum_fixed<kSteerThreadsP>(dot, red);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int c4 = threadIdx.x + q * kSteerThreadsP;
        if (4 * c4 < H) {
            const float4 vv = __ldg(reinterpret_cast<const float4*>(v) + c4);
            float4 o = make_float4(fmaf(-sF, vv.x, acc[q].x), fmaf(-sF, vv.y, acc[q].y), fmaf(-sF, vv.z, acc[q].z),
                                   fmaf(-sF, vv.w, acc[q].w));
            if (xres) {
                const int64_t e0 = (int64_t)t * H + 4 * c4;
                o = make_float4(act_at(xres, e0, D.act_bf16) + o.x, act_at(xres, e0 + 1, D.act_bf16) + o.y,
                                act_at(xres, e0 + 2, D.act_bf16) + o.z, act_at(xres, e0 + 3, D.act_bf16) + o.w);
            }
            reinterpret_cast<float4*>(out + (int64_t)t * H)[c4] = o;
        }
    }
}

// ---------------------------------------------------------------- host side
size_t gemm_smem_bytes() { return 1024 + (size_t)kGStages * (kGAStage + kGBStage) + kGSelBytes; }
// Static shared memory of the GEMM kernels (the largest of the four modes).
size_t gemm_static_smem_bytes() {
    size_t m = 0;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, k_moe_gemm<kModeGateUp, false>) == cudaSuccess && fa.sharedSizeBytes > m) m = fa.sharedSizeBytes;
    if (cudaFuncGetAttributes(&fa, k_moe_gemm<kModeDown, false>) == cudaSuccess && fa.sharedSizeBytes > m) m = fa.sharedSizeBytes;
    if (cudaFuncGetAttributes(&fa, k_moe_gemm<kModeGateUp, true>) == cudaSuccess && fa.sharedSizeBytes > m) m = fa.sharedSizeBytes;
    if (cudaFuncGetAttributes(&fa, k_moe_gemm<kModeDown, true>) == cudaSuccess && fa.sharedSizeBytes > m) m = fa.sharedSizeBytes;
    if (cudaFuncGetAttributes(&fa, k_moe_gemm<kModeShGateUp, false>) == cudaSuccess && fa.sharedSizeBytes > m) m = fa.sharedSizeBytes;
    if (cudaFuncGetAttributes(&fa, k_moe_gemm<kModeShDown, false>) == cudaSuccess && fa.sharedSizeBytes > m) m = fa.sharedSizeBytes;
    return m > sizeof(GemmSmem) ? m : sizeof(GemmSmem);
}

static PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p) return nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// Row-major bf16 [rows][cols] read as 128-row x 64-column boxes (one tensor-core half) with the 128-byte swizzle.
static cudaError_t encode_tmap(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
    const PFN_cuTensorMapEncodeTiled_v12000 fn = tmap_encoder();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {kGBK, kGHalf};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// bf16 core-matrix tiles [rows/8][cols/8][8][8] (the shared expert's layout) as a
// 3-D tensor (64-element core matrix, k chunk, 8-row group); one box is 128 rows
// x 64 columns and lands in shared memory in the same order (no swizzle).
static cudaError_t encode_tmap_core(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
    const PFN_cuTensorMapEncodeTiled_v12000 fn = tmap_encoder();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {64, cols / 8, rows / 8};
    const cuuint64_t strides[2] = {128, (cols / 8) * 128};
    const cuuint32_t box[3] = {64, kGBK / 8, kGHalf / 8};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int MODE, bool Q4>
static cudaError_t launch_gemm_t(const CUtensorMap& mapA, const CUtensorMap& mapB0, const CUtensorMap& mapB1,
                                 const GemmArgs& args, int n_sm, cudaStream_t st) {
    const size_t smem = gemm_smem_bytes();
    cudaError_t e = smem_opt_in(reinterpret_cast<const void*>(k_moe_gemm<MODE, Q4>), (int)smem);
    if (e != cudaSuccess) return e;
    k_moe_gemm<MODE, Q4><<<n_sm, kGThreads, smem, st>>>(mapA, mapB0, mapB1, args);
    return cudaGetLastError();
}
// The routed modes take the layer's expert format; the shared-expert modes have one.
template <int MODE>
static cudaError_t launch_gemm(const CUtensorMap& mapA, const CUtensorMap& mapB0, const CUtensorMap& mapB1,
                               const GemmArgs& args, int n_sm, cudaStream_t st) {
    if constexpr (MODE == kModeGateUp || MODE == kModeDown) {
        if (args.D.q4) return launch_gemm_t<MODE, true>(mapA, mapB0, mapB1, args, n_sm, st);
    }
    return launch_gemm_t<MODE, false>(mapA, mapB0, mapB1, args, n_sm, st);
}

const char* const kPrefillKernels[] = {"k_router_prefill", "k_topk_prefill", "k_hist", "k_scan", "k_scatter",
                                       "k_gather", "k_moe_gemm<gate_up>", "k_moe_gemm<down>",
                                       "k_moe_gemm<shared_gate_up>", "k_moe_gemm<shared_down>", "k_combine_prefill",
                                       "k_to_bf16"};

int prefill_launches(const Dims& D) { return D.has_shared ? (D.act_bf16 ? 11 : 12) : 9; }
const char* prefill_kernel_name(const Dims& D, int i) {
    static const int with_shared_f32[] = {11, 0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10};
    static const int with_shared_bf16[] = {0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10};
    static const int routed_only[] = {0, 1, 2, 3, 4, 5, 6, 7, 10};
    const int n = prefill_launches(D);
    if (i < 0 || i >= n) return nullptr;
    const int* order = D.has_shared ? (D.act_bf16 ? with_shared_bf16 : with_shared_f32) : routed_only;
    return kPrefillKernels[order[i]];
}

struct Marks2 {
    cudaEvent_t const* ev;
    cudaStream_t st;
    int i = 0;
    unsigned flags = 0;
    Marks2(cudaEvent_t const* e, cudaStream_t s) : ev(e), st(s) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (ev && cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
            flags = cudaEventRecordExternal;
    }
    void before() { if (ev) cudaEventRecordWithFlags(ev[2 * i], st, flags); }
    void after() {
        if (ev) cudaEventRecordWithFlags(ev[2 * i + 1], st, flags);
        ++i;
    }
};

cudaError_t launch_prefill(const Weights& W, const Dims& D, const PrefillWs& ws, const void* x, int n, float* out,
                           int n_sm, cudaStream_t st, cudaEvent_t const* ev, const int32_t* ids_in,
                           const float* wts_in) {
    cudaError_t e;
    Marks2 mk(ev, st);
    const int H = D.H, E = D.E, k = D.k, nslots = n * k;
    const int nblk = (nslots + kSortBlock - 1) / kSortBlock;
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    if (D.has_shared && !D.act_bf16) {
        const int64_t n8 = (int64_t)n * H / 8;
        mk.before();
        k_to_bf16<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(reinterpret_cast<const float*>(x), n8, ws.xb);
        mk.after();
        xb = ws.xb;
    }
    if (ids_in) {   // caller routing, copied (and checked) in place of the router's
        mk.before();
        k_routing_in<<<(unsigned)((nslots + 255) / 256), 256, 0, st>>>(ids_in, wts_in, nslots, E, ws.ids, ws.wts,
                                                                      nullptr, ws.err);
        mk.after();
        mk.before();
        mk.after();
    } else {
        mk.before();
        if ((e = launch_router_prefill(W, D, x, n, ws.logits, st)) != cudaSuccess) return e;
        mk.after();
        mk.before();
        k_topk_prefill<<<(n + 7) / 8, 256, 0, st>>>(D, ws.logits, n, ws.ids, ws.wts);
        mk.after();
    }
    mk.before();
    k_hist<<<nblk, kSortBlock, E * sizeof(int), st>>>(ws.ids, nslots, E, ws.blk_cnt);
    mk.after();
    mk.before();
    k_scan<<<1, 1024, 0, st>>>(ws.blk_cnt, nblk, E, ws.counts, ws.offs, ws.blk_off, ws.mt_prefix);
    mk.after();
    if (32 * E * sizeof(int) > 48 * 1024 &&
        (e = smem_opt_in(reinterpret_cast<const void*>(k_scatter), 32 * E * (int)sizeof(int))) != cudaSuccess)
        return e;
    mk.before();
    k_scatter<<<nblk, kSortBlock, 32 * E * sizeof(int), st>>>(ws.ids, nslots, E, ws.blk_off, ws.pos_of_slot,
                                                               ws.slot_of_pos);
    mk.after();
    mk.before();
    k_gather<<<(unsigned)((nslots + 3) / 4), 256, 0, st>>>(x, D.act_bf16, ws.slot_of_pos, nslots, k, H, ws.Xp);
    mk.after();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    GemmArgs ga{};
    ga.W = W;
    ga.D = D;
    ga.counts = ws.counts;
    ga.offs = ws.offs;
    ga.mt_prefix = ws.mt_prefix;
    ga.err = ws.err;
    ga.grid_refused = ws.grid_refused;
    CUtensorMap mA;
    // routed gate/up: A = Xp [n k][H] -> Hb [n k][I]
    if ((e = encode_tmap(&mA, ws.Xp, nslots, H)) != cudaSuccess) return e;
    ga.out_h = ws.Hb;
    mk.before();
    if ((e = launch_gemm<kModeGateUp>(mA, mA, mA, ga, n_sm, st)) != cudaSuccess) return e;
    mk.after();
    // routed down: A = Hb [n k][I] -> Y [n k][H]
    if ((e = encode_tmap(&mA, ws.Hb, nslots, D.I)) != cudaSuccess) return e;
    ga.out_y = ws.Y;
    mk.before();
    if ((e = launch_gemm<kModeDown>(mA, mA, mA, ga, n_sm, st)) != cudaSuccess) return e;
    mk.after();
    if (D.has_shared) {
        ga.n_rows = n;
        CUtensorMap mB0, mB1;
        if ((e = encode_tmap(&mA, xb, n, H)) != cudaSuccess) return e;
        if ((e = encode_tmap_core(&mB0, W.sh_gate, D.I, H)) != cudaSuccess) return e;
        if ((e = encode_tmap_core(&mB1, W.sh_up, D.I, H)) != cudaSuccess) return e;
        ga.out_h = ws.Hs;
        mk.before();
        if ((e = launch_gemm<kModeShGateUp>(mA, mB0, mB1, ga, n_sm, st)) != cudaSuccess) return e;
        mk.after();
        if ((e = encode_tmap(&mA, ws.Hs, n, D.I)) != cudaSuccess) return e;
        if ((e = encode_tmap_core(&mB0, W.sh_down, H, D.I)) != cudaSuccess) return e;
        ga.out_y = ws.Ys;
        mk.before();
        if ((e = launch_gemm<kModeShDown>(mA, mB0, mB0, ga, n_sm, st)) != cudaSuccess) return e;
        mk.after();
    }
    const int64_t n4 = (int64_t)n * H / 4;
    mk.before();
    if (ws.steer_v)
        k_combine_steer_prefill<<<(unsigned)n, kSteerThreadsP, 0, st>>>(D, ws.Ys, ws.Y, ws.wts, ws.pos_of_slot,
                                                                      ws.steer_v, ws.steer_F, ws.xres, ws.grid_refused, out);
    else
        k_combine_prefill<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(D, ws.Ys, ws.Y, ws.wts, ws.pos_of_slot, n,
                                                                        ws.xres, ws.grid_refused, out);
    mk.after();
    return cudaGetLastError();
}

// Plan of an inspection call: all n rows go to expert e (counts, offsets and
// tile prefix of the grouped GEMM).
__global__ void k_probe_plan(int E, int e, int n, int32_t* counts, int32_t* offs, int32_t* mt_prefix) {
    for (int q = threadIdx.x; q <= E; q += blockDim.x) {
        if (q < E) counts[q] = q == e ? n : 0;
        offs[q] = q <= e ? 0 : n;
        mt_prefix[q] = q <= e ? 0 : (n + kGBM - 1) / kGBM;
    }
}

// Inspection: one grouped-GEMM launch of the prefill plan on caller rows, all
// of them routed to expert e (e = -1: the shared expert).  which 0: gate/up,
// in [n][H] bf16, out [n][2I] binary32 accumulators (no SwiGLU); which 2:
// down, in [n][I] bf16, out [n][H] binary32.
cudaError_t launch_probe_gemm(const Weights& W, const Dims& D, const PrefillWs& ws, int which, int e,
                              const void* in, int n, float* out, int n_sm, cudaStream_t st) {
    cudaError_t err;
    GemmArgs ga{};
    ga.W = W;
    ga.D = D;
    ga.counts = ws.counts;
    ga.offs = ws.offs;
    ga.mt_prefix = ws.mt_prefix;
    ga.err = ws.err;
    ga.n_rows = n;
    CUtensorMap mA, mB0, mB1;
    const int K = which == 0 ? D.H : D.I;
    if ((err = encode_tmap(&mA, in, n, K)) != cudaSuccess) return err;
    if (e >= 0) {
        k_probe_plan<<<1, 256, 0, st>>>(D.E, e, n, ws.counts, ws.offs, ws.mt_prefix);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        if (which == 0) {
            ga.out_raw = out;
            return launch_gemm<kModeGateUp>(mA, mA, mA, ga, n_sm, st);
        }
        ga.out_y = out;
        return launch_gemm<kModeDown>(mA, mA, mA, ga, n_sm, st);
    }
    if (which == 0) {
        if ((err = encode_tmap_core(&mB0, W.sh_gate, D.I, D.H)) != cudaSuccess) return err;
        if ((err = encode_tmap_core(&mB1, W.sh_up, D.I, D.H)) != cudaSuccess) return err;
        ga.out_raw = out;
        return launch_gemm<kModeShGateUp>(mA, mB0, mB1, ga, n_sm, st);
    }
    if ((err = encode_tmap_core(&mB0, W.sh_down, D.H, D.I)) != cudaSuccess) return err;
    ga.out_y = out;
    return launch_gemm<kModeShDown>(mA, mB0, mB0, ga, n_sm, st);
}

// Inspection: the permutation of the prefill plan (histogram, scan, stable
// scatter) on caller ids [n][k], results in the workspace.
cudaError_t launch_permutation(const Dims& D, const PrefillWs& ws, const int32_t* ids, int n, cudaStream_t st) {
    cudaError_t e;
    const int E = D.E, nslots = n * D.k;
    const int nblk = (nslots + kSortBlock - 1) / kSortBlock;
    k_hist<<<nblk, kSortBlock, E * sizeof(int), st>>>(ids, nslots, E, ws.blk_cnt);
    k_scan<<<1, 1024, 0, st>>>(ws.blk_cnt, nblk, E, ws.counts, ws.offs, ws.blk_off, ws.mt_prefix);
    if (32 * E * sizeof(int) > 48 * 1024 &&
        (e = smem_opt_in(reinterpret_cast<const void*>(k_scatter), 32 * E * (int)sizeof(int))) != cudaSuccess)
        return e;
    k_scatter<<<nblk, kSortBlock, 32 * E * sizeof(int), st>>>(ids, nslots, E, ws.blk_off, ws.pos_of_slot,
                                                               ws.slot_of_pos);
    return cudaGetLastError();
}

// Routing only (prefill sizes): logits and top-k.
cudaError_t launch_route_prefill(const Weights& W, const Dims& D, const PrefillWs& ws, const void* x, int n,
                                 cudaStream_t st) {
    cudaError_t e = launch_router_prefill(W, D, x, n, ws.logits, st);
    if (e != cudaSuccess) return e;
    k_topk_prefill<<<(n + 7) / 8, 256, 0, st>>>(D, ws.logits, n, ws.ids, ws.wts);
    return cudaGetLastError();
}

}  // namespace ds4
