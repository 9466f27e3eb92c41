// decode.cu -- the decode plan for 1..decode_max tokens (three launches).
//
//   k_router_decode  one warp per expert row, logits in the canonical binary32
//                    order; the last CTA picks the top-k by (logit desc,
//                    index asc) and the softmax over the selected logits.
//   k_moe_decode     h = silu(W_gate x) * (W_up x), then y = W_down h, for
//                    every selected expert (read once, applied to every token
//                    that chose it) and for the shared expert.
//   k_combine_decode out = y_shared + sum_j w_j y_j in rank order (then
//                    x + that for the residual step; k_combine_steer_decode
//                    also steers: y - F v (v . y)).
//
// k_moe_decode is persistent (one CTA per SM).  A producer warp pulls tasks
// from atomic queues -- gate/up tasks (shared-expert 8-row groups and
// (expert, 32-row block) pieces; for one token from two queues, their chunks
// taken in turn), then down tasks ((expert, 32-row block) pieces, then
// shared-expert 16-row groups) -- and streams their weights into a ring of
// shared-memory stages with bulk copies (cp.async.bulk + mbarrier).  A down task first waits (bounded) until the gate/up tasks that
// produce its h have published it through completion counters.  The consumer
// warps turn the packed weights into exact small integers in registers and
// multiply them on the tensor cores with warp-level MMAs, so that the
// per-weight work is the unpacking alone; an epilogue warp sums the consumer
// warps' partial results of each task in a fixed order and finishes it:
//   IQ2 (gate, up): each 8-weight chunk becomes eight int8 values +-G by two
//     byte permutes whose selectors come from two shared-memory tables (grid
//     row -> magnitude classes, sign byte -> sign flags with the parity of
//     the eighth folded in), addressed by one byte permute each; x enters as
//     four int8 pieces of a per-token power-of-two scale (29 bits of
//     precision), the int32 products of a 32-weight group are scaled by its
//     odd integer 2s+1 in int32, and every superblock's sum is converted once
//     and scaled by d/8.
//   Q2 (down): codes become the bfloat16 numbers 1 + q/4 by a rotate, a mask
//     and two byte permutes; h enters as two bfloat16 pieces (hi, lo); each
//     16-weight sub-block's result is 4 d sc (D - S) - dmin m S with D its
//     MMA sum and S its sum of h.
//   shared expert: the bf16 weights are the MMA operand as stored; x and h
//     enter as two bfloat16 pieces.
// The MMA's eight accumulator columns hold (token, piece) pairs or, when an
// expert serves one token, different 32-weight groups (IQ2) or 16-weight
// sub-blocks (Q2) of that token, so that their scales are applied once per
// several MMAs.  k_moe_decode is launched with programmatic dependent launch:
// it starts its shared-expert tasks while the router still runs and takes the
// routing from the router's ready flag; the combine waits for it
// (griddepcontrol.wait).
#include <map>
#include <mutex>
#include <utility>

#include "ds4moe_internal.cuh"
#include "topk.cuh"

namespace ds4 {

constexpr int kMaxSlots = 128;                 // decode_max (<= 8) * top_k (<= 16)
constexpr int kStageBytes = 34816;             // 32 KB of weights + 2 KB of scales
constexpr uint32_t kTabAddr = 0x20000;          // shared address of the one- and two-token selector table
constexpr int kRE = 2;                         // router rows (warps) per CTA

// ---------------------------------------------------------------- warp MMAs
// int8 A (16 x 32, row) times int8 B (32 x 8, col), int32 accumulators.
__device__ __forceinline__ void imma_z(int (&d)[4], const uint32_t (&a)[4], uint2 b) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y), "r"(0));
}
__device__ __forceinline__ void imma(int (&d)[4], const uint32_t (&a)[4], uint2 b) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y));
}
// bf16 A (16 x 16, row) times bf16 B (16 x 8, col), binary32 accumulators.
__device__ __forceinline__ void bmma(float (&d)[4], const uint32_t (&a)[4], uint2 b) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y));
}

// Four consecutive activations (binary32, or bf16 widened exactly) from a 16-byte (8-byte) aligned index.
__device__ __forceinline__ float4 load_act4(const void* x, int64_t idx, int act_bf16) {
    if (act_bf16) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(x) + idx));
        return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u), __uint_as_float(v.y << 16),
                           __uint_as_float(v.y & 0xffff0000u));
    }
    return __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + idx));
}

__device__ __forceinline__ uint32_t bf16_bits(float v) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// Byte permute in PTX form: a selector nibble with bit 3 set replicates the sign bit of its byte.
__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// 2s + 1 for the 4-bit IQ2 group scale s of an S word in device order (bit c of s in bit 7 of byte c):
// selO (0xBA98 for the first word, 0xFEDC for the second) turns each byte into 0 or -1 by its top
// bit; the dot product with bytes (-2, -4, -8, -16) plus 1 is 2s + 1.
__device__ __forceinline__ int iq2_odd(uint32_t s0, uint32_t s1, uint32_t selO) {
    return __dp4a((int)prmt_b32(s0, s1, selO), (int)0xF0F8FCFEu, 1);
}

// ---------------------------------------------------------------- router
// One CTA per kRE expert rows; each row's tokens are split over TW warps.
// Thread 0 brings the CTA's router rows and all n token vectors into shared
// memory with two bulk copies on one mbarrier, so every CTA's rows are in
// flight at once (the 4 MB of W_r arrive in about one memory latency).  Lane
// L then runs chain L of the canonical order (columns 128 i + 4L + r, i
// ascending, r = 0..3, one fma each), the chains meet in the fixed butterfly
// (xor 16, 8, 4, 2, 1) and the bias is added once.  The last CTA to finish
// picks the top-k and, when `ready` is given, publishes it: every thread
// fences its writes, then one store with release semantics sets *ready.
template <int NT>
struct RouterCfg {
    static constexpr int TW = NT < 4 ? NT : 4;           // warps per row (token split)
    static constexpr int TPW = (NT + TW - 1) / TW;       // tokens per warp
    static constexpr int kWarps = kRE * TW;
};

template <int NT>
__global__ void __launch_bounds__(RouterCfg<NT>::kWarps * 32)
    k_router_decode(Weights W, Dims D, DecodeWs ws, const void* x, int n, uint32_t* ready) {
    using C = RouterCfg<NT>;
    constexpr int TW = C::TW, TPW = C::TPW, RW = C::kWarps;
    griddep_launch();   // the projection grid may start its shared-expert work now
    extern __shared__ __align__(128) unsigned char r_smem[];   // [kRE][H] f32 rows, then x as given [n][H]
    __shared__ uint64_t bar;
    __shared__ bool s_last;
    __shared__ float s_logits[RW][1024];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = D.H, E = D.E;
    const int e0 = blockIdx.x * kRE;
    const int nrows = E - e0 < kRE ? E - e0 : kRE;
    const float* wrows = reinterpret_cast<const float*>(r_smem);
    const unsigned char* xsm = r_smem + (size_t)kRE * H * 4;
    if (threadIdx.x == 0) {
        const uint32_t wbytes = (uint32_t)nrows * H * 4, xbytes = (uint32_t)n * H * (D.act_bf16 ? 2 : 4);
        mbar_init(&bar, 1);
        fence_barrier_init();
        mbar_arrive_expect_tx(&bar, wbytes + xbytes);
        bulk_load_plain(r_smem, W.W_r + (size_t)e0 * H, wbytes, &bar);
        griddep_wait();   // chained layers: x is the previous layer's output (no-op otherwise)
        bulk_load_plain(r_smem + (size_t)kRE * H * 4, x, xbytes, &bar);
    }
    __syncthreads();
    mbar_wait(&bar, 0, ws.err);
    const int row = warp % kRE, tw = warp / kRE;
    if (row < nrows) {
        const int e = e0 + row;
        const float* wr = wrows + (size_t)row * H + 4 * lane;
        float acc[TPW];
#pragma unroll
        for (int j = 0; j < TPW; ++j) acc[j] = 0.f;
#pragma unroll 4
        for (int i = 0; i < H / 128; ++i) {
            const float4 wv = *reinterpret_cast<const float4*>(wr + 128 * i);
#pragma unroll
            for (int j = 0; j < TPW; ++j) {
                const int t = tw + TW * j;
                if (t < n) {
                    float4 x4;
                    if (D.act_bf16) {
                        const uint2 v = *reinterpret_cast<const uint2*>(xsm + ((size_t)t * H + 128 * i + 4 * lane) * 2);
                        x4 = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                                         __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
                    } else {
                        x4 = *reinterpret_cast<const float4*>(xsm + ((size_t)t * H + 128 * i + 4 * lane) * 4);
                    }
                    acc[j] = fmaf(x4.x, wv.x, acc[j]);
                    acc[j] = fmaf(x4.y, wv.y, acc[j]);
                    acc[j] = fmaf(x4.z, wv.z, acc[j]);
                    acc[j] = fmaf(x4.w, wv.w, acc[j]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < TPW; ++j) {
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) acc[j] = acc[j] + __shfl_xor_sync(0xffffffffu, acc[j], m);
        }
        if (lane == 0) {
            const float b = W.b_r ? W.b_r[e] : 0.f;
#pragma unroll
            for (int j = 0; j < TPW; ++j) {
                const int t = tw + TW * j;
                if (t < n) ws.logits[(int64_t)t * E + e] = W.b_r ? acc[j] + b : acc[j];
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(ws.ticket, 1u);
        s_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) *ws.ticket = 0;
    for (int t = warp; t < n; t += RW)
        topk_softmax_warp(ws.logits + (int64_t)t * E, s_logits[warp], E, D.k, ws.ids + t * D.k, ws.wts + t * D.k);
    if (ready) {
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(ready), "r"(1u) : "memory");
    }
}

// Waits (bounded) until *flag is nonzero, reading it with acquire semantics.
__device__ __forceinline__ bool wait_flag(const uint32_t* flag, uint32_t* err) {
    uint64_t t0 = 0;
    for (;;) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v) return true;
        if (t0 == 0) {
            t0 = global_ns();
        } else if (global_ns() - t0 > kWaitNs) {
            set_err(err, kErrTimeout);
            return false;
        }
        __nanosleep(64);
    }
}

// Waits (bounded) until *counter >= target, reading it with acquire semantics.
__device__ __forceinline__ bool wait_ge(const uint32_t* counter, uint32_t target, uint32_t* err) {
    uint64_t t0 = 0;
    for (;;) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
        if (v >= target) return true;
        if (t0 == 0) {
            t0 = global_ns();
        } else if (global_ns() - t0 > kWaitNs) {
            set_err(err, kErrTimeout);
            return false;
        }
        __nanosleep(64);
    }
}

// Producer warp: waits (bounded) until gate/up completion counter c (0: the shared expert, 1 + u: entry u)
// has reached its target (t_sh for counter 0, t_rt for the others).  `known` caches what earlier polls saw
// (per lane, bit j: counter lane + 32 j complete), so a complete counter is not read again; a poll reads
// every unfinished counter at once, one per lane and word, instead of one load latency per task.  Orders
// the generic-proxy writes it observed before the warp's later bulk copies.
__device__ __forceinline__ bool wait_deps_warp(const uint32_t* ctr, int c, int ncnt, uint32_t t_sh, uint32_t t_rt,
                                               uint32_t& known, uint32_t* err) {
    const int lane = threadIdx.x & 31;
    uint64_t t0 = 0;
    for (;;) {
        const uint32_t kb = __shfl_sync(0xffffffffu, known, c & 31);
        if ((kb >> (c >> 5)) & 1u) return true;
        if (t0 != 0) __nanosleep(32);
#pragma unroll
        for (int j = 0; j < 5; ++j) {
            const int idx = lane + 32 * j;
            if (idx < ncnt && !((known >> j) & 1u)) {
                uint32_t v;
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr + idx) : "memory");
                if (v >= (idx == 0 ? t_sh : t_rt)) known |= 1u << j;
            }
        }
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncwarp();
        const uint64_t now = __shfl_sync(0xffffffffu, (unsigned long long)global_ns(), 0);
        if (t0 == 0) {
            t0 = now;
        } else if (now - t0 > kWaitNs) {
            if (lane == 0) set_err(err, kErrTimeout);
            return false;
        }
    }
}

// ---------------------------------------------------------------- routing table
// Routed tasks' experts ("entries") in ascending expert order, each with the
// slots (t * k + j) that chose it in increasing slot order, at most tpb slots
// per entry (an expert chosen by more tokens gets several entries, each
// reading its weights once).  Built by one warp.  Probe calls (probe 1) route
// every token to expert probe_e through slot t * k; probe 2 has no entries.
struct Routing {
    int nu;
    int uniq[kMaxSlots];
    int ustart[kMaxSlots + 1];
    int slot[kMaxSlots];
    int ids[kMaxSlots];
    int first[kMaxSlots];
    int rank[kMaxSlots];
    int pos[kMaxSlots];
};

__device__ void build_routing_warp(Routing& R, const int32_t* ids, int n, int k, int tpb, int probe, int probe_e) {
    const int lane = threadIdx.x & 31, nk = n * k;
    if (probe) {
        if (lane == 0) {
            const int nu = probe == 1 ? (n + tpb - 1) / tpb : 0;
            for (int u = 0; u < nu; ++u) {
                R.uniq[u] = probe_e;
                R.ustart[u] = u * tpb;
            }
            R.ustart[nu] = n;
            for (int t = 0; t < n; ++t) R.slot[t] = t * k;
            R.nu = nu;
        }
        __syncwarp();
        return;
    }
    for (int s = lane; s < nk; s += 32) R.ids[s] = __ldcg(ids + s);
    __syncwarp();
    for (int s = lane; s < nk; s += 32) {
        const int e = R.ids[s];
        int first = 1, pos = 0;
        for (int q = 0; q < s; ++q)
            if (R.ids[q] == e) { first = 0; ++pos; }
        R.first[s] = first;
        R.pos[s] = pos;
    }
    __syncwarp();
    for (int s = lane; s < nk; s += 32) {
        const int e = R.ids[s];
        int rank = 0, cnt = 0;
        for (int q = 0; q < nk; ++q) {
            rank += (R.first[q] && R.ids[q] < e);
            cnt += R.ids[q] == e;
        }
        R.rank[s] = rank;
        if (R.first[s]) {
            R.uniq[rank] = e;
            R.ustart[rank + 1] = cnt;
        }
    }
    __syncwarp();
    if (lane == 0) {
        int nu = 0;
        for (int s = 0; s < nk; ++s) nu += R.first[s];
        R.nu = nu;
        R.ustart[0] = 0;
        for (int u = 0; u < nu; ++u) R.ustart[u + 1] += R.ustart[u];
    }
    __syncwarp();
    for (int s = lane; s < nk; s += 32) R.slot[R.ustart[R.rank[s]] + R.pos[s]] = s;
    __syncwarp();
    if (lane == 0) {   // split the entries into runs of at most tpb slots (scratch: first = experts, rank = starts)
        const int nu = R.nu;
        for (int u = 0; u <= nu; ++u) R.rank[u] = R.ustart[u];
        for (int u = 0; u < nu; ++u) R.first[u] = R.uniq[u];
        int m = 0;
        for (int u = 0; u < nu; ++u)
            for (int s = R.rank[u]; s < R.rank[u + 1]; s += tpb) {
                R.uniq[m] = R.first[u];
                R.ustart[m] = s;
                ++m;
            }
        R.ustart[m] = nk;
        R.nu = m;
    }
    __syncwarp();
}

// ---------------------------------------------------------------- pipeline state
struct ChunkInfo {
    int task;      // -1: no more work
    int chunk;     // chunk index within the task
    int nchunk;    // chunks of the task
    int lo, cnt;   // routed: first k step (64 columns) of the chunk and how many; shared: first column, columns
};

struct Pipe {
    uint64_t full[4];
    uint64_t empty[4];
    uint64_t cons;        // barrier of the consumer warps (task epilogues)
    ChunkInfo info[4];
    int abort;            // set after a timed-out wait: every loop leaves
};

__device__ void pipe_init(Pipe& P, int NS, int CW) {
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&P.full[s], 1);
            mbar_init(&P.empty[s], CW);
        }
        mbar_init(&P.cons, CW);
        P.abort = 0;
        fence_barrier_init();
    }
}

__device__ __forceinline__ bool aborted(const Pipe& P) { return *(volatile const int*)&P.abort != 0; }
__device__ __forceinline__ void set_abort(Pipe& P) { *(volatile int*)&P.abort = 1; }

// Bounded barrier of the consumer warps (instead of bar.sync, which
// cannot time out).  Returns false after a timeout.
__device__ __forceinline__ bool cons_sync(Pipe& P, uint32_t& phase, uint32_t* err) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&P.cons);
    const bool ok = mbar_wait(&P.cons, phase, err);
    phase ^= 1u;
    if (!ok) set_abort(P);
    return ok;
}

// Producer: wait until the last NS issued copies have landed (bounded), then
// publish the stop marker.  Leaves no bulk copy in flight.
__device__ void producer_finish(Pipe& P, uint32_t it, int NS, uint32_t* err) {
    const int lane = threadIdx.x & 31;
    const uint32_t j0 = it > (uint32_t)NS ? it - NS : 0;
    for (uint32_t j = j0; j < it; ++j) mbar_wait(&P.full[j % NS], (j / NS) & 1, err);
    const int s = it % NS;
    if (!aborted(P)) {
        if (!mbar_wait(&P.empty[s], ((it / NS) & 1) ^ 1, err)) set_abort(P);
    }
    if (lane == 0) {
        P.info[s].task = -1;
        mbar_arrive(&P.full[s]);
    }
    __syncwarp();
}

// Position of column c of h in the routed h layout ([I/64][2 pieces][64]
// per slot): inside each 16-column block, column 4e + c4 sits at 4 c4 + e, the
// order in which the down kernel's MMA fragments read the codes of a block.
__device__ __forceinline__ int hrt_index(int c, int piece) {
    const int w = c & 63;
    return ((c >> 6) * 2 + piece) * 64 + (w & ~15) + 4 * (w & 3) + ((w >> 2) & 3);
}
__device__ __forceinline__ int hsh_index(int c, int piece) { return ((c >> 6) * 2 + piece) * 64 + (c & 63); }

// ---------------------------------------------------------------- task reductions
// The consumer warps of a projection kernel split every task's columns, so a task ends with a sum over
// the warps.  Each consumer warp writes its partial sums into reduction buffer b = (its task count) % NB
// and counts itself in; a separate epilogue warp takes the buffers in order, sums the partials in warp
// order (deterministic), finishes the task (activation, stores, completion count) and frees the buffer
// for its next use.  The consumers thus never wait on a task's final reduction, only (rarely) on a
// buffer that the epilogue warp has not freed yet.
constexpr int kMaxRedBufs = 8;
struct RedRing {
    int cnt[kMaxRedBufs];     // consumer warps that wrote their partials into buffer b
    int task[kMaxRedBufs];    // the task whose partials buffer b holds
    int freed[kMaxRedBufs];   // uses of buffer b that the epilogue warp has finished
    int exits;                // consumer warps that left their loop
    int ntasks;               // tasks the consumer warps finished (read once exits == consumer warps)
};

__device__ __forceinline__ int ld_shared_volatile(const int* p) { return *reinterpret_cast<const volatile int*>(p); }

// Consumer side: waits (bounded) until buffer b is free for its use number `use`.
__device__ __forceinline__ bool ring_acquire(RedRing& R, int b, int use, uint32_t* err) {
    if (ld_shared_volatile(&R.freed[b]) >= use) return true;
    const uint64_t t0 = global_ns();
    while (ld_shared_volatile(&R.freed[b]) < use) {
        if (global_ns() - t0 > kWaitNs) {
            set_err(err, kErrTimeout);
            return false;
        }
        __nanosleep(32);
    }
    return true;
}

// Consumer side, lane 0 after the warp's partials are written: buffer b holds task `task`.
__device__ __forceinline__ void ring_publish(RedRing& R, int b, int task) {
    R.task[b] = task;
    __threadfence_block();
    atomicAdd(&R.cnt[b], 1);
}

// Consumer side, lane 0 when the warp leaves its loop after finishing `ntask` tasks.
__device__ __forceinline__ void ring_exit(RedRing& R, int ntask) {
    atomicMax(&R.ntasks, ntask);
    __threadfence_block();
    atomicAdd(&R.exits, 1);
}

// Epilogue side (whole warp): waits (bounded) until buffer j % nb holds the partials of every consumer
// warp; false once the consumers have left and buffer j will not be filled.
__device__ __forceinline__ bool ring_take(RedRing& R, uint32_t j, int nb, int cw, uint32_t* err) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) {
        const int b = (int)(j % nb);
        uint64_t t0 = 0;
        for (;;) {
            if (ld_shared_volatile(&R.cnt[b]) == cw) { ok = 1; break; }
            if (ld_shared_volatile(&R.exits) == cw && (int)j >= ld_shared_volatile(&R.ntasks)) break;
            if (t0 == 0) {
                t0 = global_ns();
            } else if (global_ns() - t0 > kWaitNs) {
                set_err(err, kErrTimeout);
                break;
            }
            __nanosleep(32);
        }
        __threadfence_block();
    }
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Epilogue side (whole warp) after finishing buffer j: free it for its next use.
__device__ __forceinline__ void ring_free(RedRing& R, uint32_t j, int nb) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
        const int b = (int)(j % nb);
        R.cnt[b] = 0;
        __threadfence_block();
        R.freed[b] = (int)(j / nb) + 1;
    }
    __syncwarp();
}

// x (n tokens of H) as four int8 pieces per value, [n][4][H] bytes: v = x f1 f2 (|v| < 128), piece p
// = trunc of the remaining fraction times 128^p.  quantize4 writes values i..i+3 of token tk.
__device__ __forceinline__ void quantize4(float4 xv, float f1, float f2, unsigned char* xq, int H, int tk, int i) {
    const float vv[4] = {xv.x, xv.y, xv.z, xv.w};
    uint32_t pw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float v = vv[j] * f1 * f2;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float tv = truncf(v);
            pw[p] |= ((uint32_t)(int)tv & 0xffu) << (8 * j);
            v = (v - tv) * 128.f;
        }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) *reinterpret_cast<uint32_t*>(xq + (size_t)(tk * 4 + p) * H + i) = pw[p];
}
// Every token's values, threads tid of nthreads, four values each.
__device__ __forceinline__ void quantize_x(const void* x, int act_bf16, int n, int H, const float (*s_f)[2],
                                           unsigned char* xq, int tid, int nthreads) {
    for (int q = tid * 4; q < n * H; q += nthreads * 4) {
        const int tk = q / H, i = q - tk * H;
        quantize4(load_act4(x, (int64_t)tk * H + i, act_bf16), s_f[tk][0], s_f[tk][1], xq, H, tk, i);
    }
}

// Barrier 1 of the threads that run the projection kernel's prologue.
__device__ __forceinline__ void prologue_sync(int nthreads) {
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- gate/up
template <int NT, bool Q4 = false>
struct GateUpCfg {
    static constexpr int CW = 8;                                  // consumer warps
    // stages: 4-bit layers have no selector table, and one or two tokens take four stages of 37 KB
    // (16 k steps of gate and up codes with their scales) to keep more bytes in flight
    static constexpr int NS = NT <= 2 && Q4 ? 4 : NT <= 4 ? 3 : 2;
    static constexpr int kStage = Q4 && NT <= 4 ? 37888 : kStageBytes;
    // selector tables: ROWS form (one or two tokens): 256 rows of 256 B, bytes 0..127 of row r the
    // class selectors of grid row r, bytes 128..255 the sign selectors of S byte r (signs r & 127),
    // 32 copies each (one per lane), so that one byte-permute of a payload word and the lane's offset
    // is the row's address; otherwise tsel [256][R] and tsgn [128][R] with R interleaved copies
    static constexpr bool kRows = NT <= 2;
    static constexpr int R = NT == 4 ? 16 : 8;
    static constexpr int TPB = NT == 1 ? 1 : 2;                   // tokens of one routed entry
    static constexpr int kThreads = (CW + 2) * 32;                // + producer warp + epilogue warp
    static constexpr int kTabWords = kRows ? 256 * 64 : (256 + 128) * R;
    // task reductions: a ring of NB buffers of [warp][kRedPer] partial sums (routed: TPB tokens x 64
    // rows; shared: up to 8 tokens x 16 rows)
    static constexpr int NB = NT == 8 ? NS + 1 : NS + 2;
    static constexpr int kRedPer = NT == 1 ? 64 : 128;
    static constexpr int kRedFloats = NB * CW * kRedPer;
    // one token: x's int8 pieces get their own buffer, made in the prologue; otherwise they replace the
    // bf16 pieces once the shared-expert tasks are done
    static constexpr bool kSplitX = NT == 1;
};

// The IQ2 chunk of one thread (8 weights, grid row a from byte t of the
// index word, signs in byte t of S) as int8 +-G: weights 0..3 in lo, 4..7 in
// hi.  The selector's nibble i is the magnitude class of weight i plus 4 for
// a negative sign; (clo, chi) hold the four magnitudes and their negatives.
// Rows form: tb = the table's shared address, lbA / lbB = this lane's byte
// offset in the class / sign half of a row, selT puts byte t of the word in
// byte 1 of the offset.
__device__ __forceinline__ void iq2_chunk_rows(uint32_t idx, uint32_t S, uint32_t tb, uint32_t lbA, uint32_t lbB,
                                               uint32_t selT, uint32_t clo, uint32_t chi, uint32_t& lo,
                                               uint32_t& hi) {
    const uint32_t sel = ld_shared_u32(tb + __byte_perm(idx, lbA, selT)) | ld_shared_u32(tb + __byte_perm(S, lbB, selT));
    lo = __byte_perm(clo, chi, sel);
    hi = __byte_perm(clo, chi, sel >> 16);
}
// Interleaved form: tsel / tsgn point at this lane's copy (R words per entry).
template <int R>
__device__ __forceinline__ void iq2_chunk_s8(uint32_t idx, uint32_t S, uint32_t selA, int t8, const uint32_t* tsel,
                                             const uint32_t* tsgn, uint32_t clo, uint32_t chi, uint32_t& lo,
                                             uint32_t& hi) {
    const uint32_t a = __byte_perm(idx, 0u, selA);
    const uint32_t sg = (S >> t8) & 127u;
    const uint32_t sel = tsel[a * R] | tsgn[sg * R];
    lo = __byte_perm(clo, chi, sel);
    hi = __byte_perm(clo, chi, sel >> 16);
}

// Q4 down codes (mode-1 order) of rows g (w0) and g + 8 (w1), one word = two
// 16-column groups: the bf16 A fragments of those groups, each element
// 1 + q/16 (exact: 0x3F80 | q << 3).
__device__ __forceinline__ void q4_down_frags(uint32_t w0, uint32_t w1, uint32_t (&a)[4], uint32_t (&b)[4]) {
    constexpr uint32_t M = 0x00780078u, ONE = 0x3F803F80u;
    a[0] = ((w0 << 3) & M) | ONE;
    a[1] = ((w1 << 3) & M) | ONE;
    a[2] = ((w0 >> 1) & M) | ONE;
    a[3] = ((w1 >> 1) & M) | ONE;
    b[0] = ((w0 >> 5) & M) | ONE;
    b[1] = ((w1 >> 5) & M) | ONE;
    b[2] = ((w0 >> 9) & M) | ONE;
    b[3] = ((w1 >> 9) & M) | ONE;
}

// Per consumer thread state of the gate/up kernel's tasks.
template <int NT>
struct GateUpAcc {
    static constexpr int TG = (NT + 3) / 4;   // token groups of four (shared tasks)
    float sh[TG][2][4];                       // shared task: [token group][gate, up][fragment] (rows g only)
    float rt[GateUpCfg<NT>::TPB][4][2];       // routed task: [token][tile][row g, g + 8]
};

// ---------------------------------------------------------------- down projection pieces
// k steps (64 columns) per routed down chunk for an entry of ns slots: codes,
// scales (step_bytes per step: 640 for Q2, 1152 for Q4), (d, dmin) and the
// slots' h pieces (and per-16 sums) for those columns must fit one stage of
// stage_bytes.
__device__ __forceinline__ int down_chunk_ksteps(int nkt, int nsb, int ns, int step_bytes, int stage_bytes) {
    // the largest of 32, 16, 8, 4 that divides the k steps (I / 64: a multiple of 4 for I >= 256)
    int ck = nkt % 32 == 0 ? 32 : nkt % 16 == 0 ? 16 : nkt % 8 == 0 ? 8 : nkt % 4 == 0 ? 4 : nkt;
    for (; ck > 1 && ck % 2 == 0; ck >>= 1) {
        const int nsbc = nsb > 1 ? (ck + 3) / 4 : 1;
        if (ck * step_bytes + nsbc * 128 + ns * ck * 272 <= stage_bytes) break;
    }
    return ck;
}

template <int NT>
struct DownAcc {
    static constexpr int TG = (NT + 3) / 4;
    float sh[TG][4];                           // shared task: [token group][fragment]
    float rt[GateUpCfg<NT>::TPB][2][2];          // routed task: [token][tile][row g, g + 8]
};


// Q4: the routed experts' three matrices are Q4 blocks (no grid tables; x's
// per-32-column sums for the min terms).
template <int NT, bool Q4>
__global__ void __launch_bounds__(GateUpCfg<NT>::kThreads, 1)
    k_moe_decode(Weights W, Dims D, DecodeWs ws, const void* x, int n) {
    using C = GateUpCfg<NT, Q4>;
    constexpr int NS = C::NS, CW = C::CW, R = C::R, TPB = C::TPB, kThreads = C::kThreads;
    constexpr int kTab = Q4 ? 0 : C::kTabWords;
    constexpr int kStage = C::kStage;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    // one or two tokens (rows table): the table sits at shared address kTabAddr, after the stages and the
    // reduction ring, so that one byte permute (grid row, lane offset, the address's upper bytes) is a
    // row's address with no add; x's buffers follow it
    constexpr bool kAbs = !Q4 && C::kRows;
    const uint32_t base = smem_addr(smem_raw);
    uint32_t* tsel = kAbs ? reinterpret_cast<uint32_t*>(smem_raw + (kTabAddr - base))
                          : reinterpret_cast<uint32_t*>(smem_raw);                // rows [256][64] or [256][R]
    uint32_t* tsgn = tsel + 256 * R;                                             // [128][R] (interleaved form)
    unsigned char* stages = kAbs ? smem_raw : smem_raw + 4 * kTab;               // NS x kStage
    float* red = reinterpret_cast<float*>(stages + NS * kStage);                 // kRedFloats
    unsigned char* xbuf = kAbs ? reinterpret_cast<unsigned char*>(tsel + 256 * 64)
                               : reinterpret_cast<unsigned char*>(red + C::kRedFloats);  // n x H x 4 bytes: bf16 pieces
    unsigned char* xq = C::kSplitX ? xbuf + (size_t)n * D.H * 4 : xbuf;          // int8 pieces
    unsigned char* zero = xq + (size_t)n * D.H * 4;                              // 64 bytes of zeros
    float* xsum = reinterpret_cast<float*>(zero + 64);                           // Q4: [n][H / 32] sums of x
    __shared__ Pipe P;
    __shared__ Routing Rt;
    __shared__ int s_last, s_refused;
    __shared__ uint32_t s_cand[2];
    __shared__ float s_tokmax[8];
    __shared__ float s_cs[8][4];
    __shared__ float s_f[8][2];
    __shared__ RedRing RR;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int H = D.H, I = D.I, k = D.k;
    const int nkt = H / 64, nsb = H / 256;
    // which projections this call runs: the forward runs both; the inspection probes run one
    const bool do_gu = (ws.stages & 1) != 0, do_dn = (ws.stages & 2) != 0;
    const int n_sh = !do_gu || ws.probe == 1 ? 0 : (D.has_shared ? I / 8 : 0);   // shared tasks: 8 rows of gate and up
    const int rb_per_e = I / 32;
    // k steps (64 columns) per routed chunk: the largest of 32, 16, 8, 4 that divides H / 64 and fits a
    // stage (Q4: 16 with the 37 KB stage, else 8)
    const int ck_rt = (!Q4 && nkt % 32 == 0) ? 32
                      : ((!Q4 || kStage >= 37888) && nkt % 16 == 0) ? 16
                      : nkt % 8 == 0 ? 8 : 4;
    const int nch_rt = nkt / ck_rt;
    const int kcs = H < 1024 ? H : 1024;              // columns per shared chunk
    const int nch_sh = H / kcs;
    // down projection: tasks (entry, 32-row block) in entry order, then tasks of 16 shared-expert rows,
    // numbered after the gate/up tasks; a task first waits until the gate/up tasks producing its h are
    // done (the first entries' h is the first ready; the shared expert's h needs every shared gate/up
    // task, some of which come last)
    const int dnkt = I / 64, dnsb = I >= 256 ? I / 256 : 1;
    const int dn_sh = !do_dn || ws.probe == 1 ? 0 : (D.has_shared ? H / 16 : 0);
    const int drb = H / 32;
    const int dkcs = I < 512 ? I : 512;   // columns per shared-expert chunk
    const int dnch_sh = I / dkcs;

    __shared__ uint64_t tab_bar;
    if (kAbs) {
        // the layout needs the dynamic shared memory to reach past the table (the launch asks for it, counting
        // at least 4 KB of static shared memory before it): refuse the call instead of running out of it
        uint32_t dyn;
        asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
        const uint32_t need_end = kTabAddr + 256 * 64 * 4 + (C::kSplitX ? 2u : 1u) * n * D.H * 4 + 64;
        const uint32_t low_end = base + NS * kStage + 4 * C::kRedFloats;
        if (low_end > kTabAddr || need_end > base + dyn) {
            if (tid == 0) set_err(ws.err, kErrBounds);
            return;
        }
    }
    pipe_init(P, NS, CW);
    if (!Q4 && C::kRows && tid == 0) {
        // the selector table: one bulk copy, waited for at the end of the prologue
        mbar_init(&tab_bar, 1);
        fence_barrier_init();
        mbar_arrive_expect_tx(&tab_bar, 256 * 64 * 4);
        bulk_load_plain(tsel, W.gtab_rows, 256 * 64 * 4, &tab_bar);
    }
    __syncthreads();   // the pipeline's barriers are initialized
    // ---- prologue, on every warp but the producer's (which starts streaming at once): ptid / kPro
    // number its threads
    constexpr int kPro = kThreads - 32;
    const int ptid = tid < CW * 32 ? tid : tid - 32;
    if (warp != CW) {
    if (ws.chain_wait) {
        // chained layers: x is the previous layer's output, complete once its combine CTAs have counted
        if (tid == 0 && !wait_ge(ws.chain_wait, ws.chain_target, ws.err)) set_abort(P);
        prologue_sync(kPro);
    }
    // ---- grid tables (made when the grid was loaded)
    if (Q4 || C::kRows) {
    } else {
        for (int i = ptid; i < 384 * R; i += kPro) tsel[i] = __ldg(W.gtab + i / R);   // tsgn follows tsel
    }
    if (tid < 4) reinterpret_cast<uint4*>(zero)[tid] = make_uint4(0, 0, 0, 0);
    if (tid < kMaxRedBufs) RR.cnt[tid] = RR.task[tid] = RR.freed[tid] = 0;
    if (tid == 0) RR.exits = RR.ntasks = 0;
    if (tid == 0) {
        s_cand[0] = Q4 ? 0u : __ldg(W.gtab + 384);
        s_cand[1] = Q4 ? 0u : __ldg(W.gtab + 385);
        s_refused = Q4 ? 0 : (int)__ldg(W.gtab + 386);
        if (s_refused) set_err(ws.err, kErrGrid);
        if (blockIdx.x == 0) *ws.grid_refused = (uint32_t)s_refused;
    }
    // ---- token maxima and int8-piece factors (routed tasks), bf16 pieces of x (shared tasks)
    {
        float mx[NT];
#pragma unroll
        for (int q = 0; q < NT; ++q) mx[q] = 0.f;
        // one token, H <= 16 kPro: this thread's values stay in registers for the int8 pieces
        constexpr int kXr = 4;
        static_assert(kPro % 8 == 0, "32-column blocks of x per eight threads");
        const bool xreg = C::kSplitX && H <= kXr * 4 * kPro;
        float4 xr[kXr];
#pragma unroll
        for (int j = 0; j < kXr; ++j) xr[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (xreg && do_gu) {
#pragma unroll
            for (int j = 0; j < kXr; ++j) {
                const int i = (ptid + j * kPro) * 4;
                if (i < H) {
                    xr[j] = load_act4(x, i, D.act_bf16);
                    const float4 v = xr[j];
                    mx[0] = fmaxf(mx[0], fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
                    if (n_sh > 0) {
                        const uint32_t h0 = bf16_bits(v.x), h1 = bf16_bits(v.y), h2 = bf16_bits(v.z), h3 = bf16_bits(v.w);
                        const uint32_t l0 = bf16_bits(v.x - __uint_as_float(h0 << 16));
                        const uint32_t l1 = bf16_bits(v.y - __uint_as_float(h1 << 16));
                        const uint32_t l2 = bf16_bits(v.z - __uint_as_float(h2 << 16));
                        const uint32_t l3 = bf16_bits(v.w - __uint_as_float(h3 << 16));
                        *reinterpret_cast<uint2*>(xbuf + (size_t)i * 2) = make_uint2(h0 | (h1 << 16), h2 | (h3 << 16));
                        *reinterpret_cast<uint2*>(xbuf + ((size_t)H + i) * 2) = make_uint2(l0 | (l1 << 16), l2 | (l3 << 16));
                    }
                }
                if (Q4) {
                    // the 32-column sums: eight consecutive threads hold one 32-column block
                    // (kPro is a multiple of 8)
                    float sx = i < H ? (xr[j].x + xr[j].y) + (xr[j].z + xr[j].w) : 0.f;
                    sx += __shfl_xor_sync(0xffffffffu, sx, 1);
                    sx += __shfl_xor_sync(0xffffffffu, sx, 2);
                    sx += __shfl_xor_sync(0xffffffffu, sx, 4);
                    if (i < H && (lane & 7) == 0) xsum[i >> 5] = sx;
                }
            }
        }
        for (int i = ptid * 4; !xreg && do_gu && i < H; i += kPro * 4) {
#pragma unroll
            for (int q = 0; q < NT; ++q) {
                if (q < n) {
                    const float4 v = load_act4(x, (int64_t)q * H + i, D.act_bf16);
                    mx[q] = fmaxf(mx[q], fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
                    if (n_sh > 0) {
                        const uint32_t h0 = bf16_bits(v.x), h1 = bf16_bits(v.y), h2 = bf16_bits(v.z), h3 = bf16_bits(v.w);
                        const uint32_t l0 = bf16_bits(v.x - __uint_as_float(h0 << 16));
                        const uint32_t l1 = bf16_bits(v.y - __uint_as_float(h1 << 16));
                        const uint32_t l2 = bf16_bits(v.z - __uint_as_float(h2 << 16));
                        const uint32_t l3 = bf16_bits(v.w - __uint_as_float(h3 << 16));
                        *reinterpret_cast<uint2*>(xbuf + ((size_t)q * 2 * H + i) * 2) = make_uint2(h0 | (h1 << 16), h2 | (h3 << 16));
                        *reinterpret_cast<uint2*>(xbuf + ((size_t)(q * 2 + 1) * H + i) * 2) =
                            make_uint2(l0 | (l1 << 16), l2 | (l3 << 16));
                    }
                }
            }
        }
#pragma unroll
        for (int q = 0; q < NT; ++q) {
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) mx[q] = fmaxf(mx[q], __shfl_xor_sync(0xffffffffu, mx[q], m));
        }
        if (tid < 8) s_tokmax[tid] = 0.f;
        prologue_sync(kPro);
        if (lane == 0) {
#pragma unroll
            for (int q = 0; q < NT; ++q)
                if (q < n) atomicMax(reinterpret_cast<int*>(&s_tokmax[q]), __float_as_int(mx[q]));
        }
        prologue_sync(kPro);
        if (tid < n) {
            // x 2^(7-e) has |v| < 128 (e: the exponent of the token's largest |x|); the scaling is split in
            // two factors so that neither overflows; piece p weighs 2^(e - 7 - 7p)
            int e = 0;
            frexpf(s_tokmax[tid], &e);
            const int sh1 = (7 - e) / 2, sh2 = 7 - e - sh1;
            s_f[tid][0] = ldexpf(1.f, sh1);
            s_f[tid][1] = ldexpf(1.f, sh2);
#pragma unroll
            for (int p = 0; p < 4; ++p) s_cs[tid][p] = s_tokmax[tid] > 0.f ? ldexpf(1.f, e - 7 - 7 * p) : 0.f;
        }
        prologue_sync(kPro);
        if (Q4 && do_gu && !xreg) {
            // sums of x over each 32-column sub-block (the min terms)
            for (int i = ptid; i < n * (H / 32); i += kPro) {
                const int tk = i / (H / 32), j = i - tk * (H / 32);
                float sx = 0.f;
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float4 v = load_act4(x, (int64_t)tk * H + 32 * j + c, D.act_bf16);
                    sx += (v.x + v.y) + (v.z + v.w);
                }
                xsum[i] = sx;
            }
            if (!C::kSplitX) prologue_sync(kPro);
        }
        if (C::kSplitX && do_gu) {
            if (xreg) {
#pragma unroll
                for (int j = 0; j < kXr; ++j) {
                    const int i = (ptid + j * kPro) * 4;
                    if (i < H) quantize4(xr[j], s_f[0][0], s_f[0][1], xq, H, 0, i);
                }
            } else {
                quantize_x(x, D.act_bf16, n, H, s_f, xq, ptid, kPro);
            }
            prologue_sync(kPro);
        }
    }
    if (!Q4 && C::kRows && !mbar_wait(&tab_bar, 0, ws.err)) set_abort(P);
    }
    // the producer reads the grid's verdict itself (the prologue's copy is not yet written)
    const bool refused = warp == CW ? (!Q4 && __ldg(W.gtab + 386) != 0) : s_refused != 0;

    if (warp == CW) {
        // ------------------------------------------------ producer warp
        const uint64_t pol = policy_evict_first();
        uint32_t it = 0;
        bool routed = false;
        int total = 0x7fffffff;
        int d_total = 0;
        uint32_t dknown = 0;   // gate/up completion counters seen complete (wait_deps_warp)
        auto route = [&]() {
            build_routing_warp(Rt, ws.ids, n, k, TPB, ws.probe == 1 ? 1 : (ws.probe == 2 ? 2 : 0), ws.probe_e);
            routed = true;
            total = n_sh + (do_gu ? Rt.nu * rb_per_e : 0);
            d_total = dn_sh + (do_dn ? Rt.nu * drb : 0);
        };
        // one chunk c of gate/up task `task` (shared expert below n_sh, routed above) into the next stage
        auto issue_gu = [&](int task, int c) -> bool {
            const bool sh = task < n_sh;
            const int nch = sh ? nch_sh : nch_rt;
            const int s = it % NS;
            const uint32_t ph = (it / NS) & 1;
            if (!mbar_wait(&P.empty[s], ph ^ 1, ws.err)) { set_abort(P); return false; }
            if (lane == 0) {
                unsigned char* st = stages + s * kStage;
                if (sh) {
                    // one 8-row group of the gate and of the up matrix (core-matrix tiles), columns
                    // c*kcs .. +kcs
                    const int kc0 = c * kcs;
                    const uint32_t bytes = kcs * 16;
                    const size_t off = ((size_t)task * (H / 8) + kc0 / 8) * 64;   // elements
                    P.info[s] = ChunkInfo{task, c, nch, kc0, kcs};
                    mbar_arrive_expect_tx(&P.full[s], 2 * bytes);
                    bulk_load(st, W.sh_gate + off, bytes, &P.full[s], pol);
                    bulk_load(st + bytes, W.sh_up + off, bytes, &P.full[s], pol);
                } else {
                    const int tt = task - n_sh, u = tt / rb_per_e, rb = tt % rb_per_e;
                    const int e = Rt.uniq[u];
                    const int kt0 = c * ck_rt;
                    P.info[s] = ChunkInfo{task, c, nch, kt0, ck_rt};
                    if (Q4) {
                        // gate codes, up codes [ck][32][32 B], their scale words [ck][32], (d, dmin)
                        // words [ck / 4][32]
                        const uint32_t cb = ck_rt * 1024, sb = ck_rt * 128, db = (ck_rt / 4) * 128;
                        const size_t qoff = (size_t)e * W.q4_q_stride + ((size_t)rb * nkt + kt0) * 1024;
                        const size_t soff = (size_t)e * W.q4_sc_stride + ((size_t)rb * nkt + kt0) * 32;
                        const size_t doff = (size_t)e * W.q4_dd_stride + ((size_t)rb * nsb + kt0 / 4) * 32;
                        mbar_arrive_expect_tx(&P.full[s], 2 * (cb + sb + db));
                        bulk_load(st, W.gate_qs + qoff, cb, &P.full[s], pol);
                        bulk_load(st + cb, W.up_qs + qoff, cb, &P.full[s], pol);
                        bulk_load(st + 2 * cb, W.gate_sc4 + soff, sb, &P.full[s], pol);
                        bulk_load(st + 2 * cb + sb, W.up_sc4 + soff, sb, &P.full[s], pol);
                        bulk_load(st + 2 * (cb + sb), W.gate_dd4 + doff, db, &P.full[s], pol);
                        bulk_load(st + 2 * (cb + sb) + db, W.up_dd4 + doff, db, &P.full[s], pol);
                    } else {
                        const uint32_t pb = ck_rt * 512, db = ck_rt * 16;
                        const size_t qoff = (size_t)e * W.iq2_qs_stride + ((size_t)rb * nkt + kt0) * 512;
                        const size_t doff = (size_t)e * W.iq2_d_stride + ((size_t)rb * nsb + kt0 / 4) * 32;
                        mbar_arrive_expect_tx(&P.full[s], 2 * pb + 2 * db);
                        bulk_load(st, W.gate_qs + qoff, pb, &P.full[s], pol);
                        bulk_load(st + pb, W.up_qs + qoff, pb, &P.full[s], pol);
                        bulk_load(st + 2 * pb, W.gate_d + doff, db, &P.full[s], pol);
                        bulk_load(st + 2 * pb + db, W.up_d + doff, db, &P.full[s], pol);
                    }
                }
            }
            __syncwarp();
            ++it;
            return true;
        };
        // down task dt: waits (bounded) for the gate/up tasks that produce its h, then streams its chunks
        auto run_down = [&](int dt) -> bool {
            const int nd_rt = do_dn ? Rt.nu * drb : 0;
            const bool dsh = dt >= nd_rt;
            const int dts = dt - nd_rt;   // shared-expert down task
            int u = 0, rb = 0, ns = 0, ck = 0;
            if (!dsh) {
                u = dt / drb;
                rb = dt % drb;
                ns = Rt.ustart[u + 1] - Rt.ustart[u];
                ck = down_chunk_ksteps(dnkt, dnsb, ns, Q4 ? 1152 : 640, kStage);
            }
            const int nch = dsh ? dnch_sh : dnkt / ck;
            if (!ws.probe &&
                !wait_deps_warp(ws.gu_done, dsh ? 0 : 1 + u, 1 + Rt.nu, (uint32_t)(I / 8), (uint32_t)(I / 32), dknown,
                                ws.err)) {
                set_abort(P);
                return false;
            }
            for (int c = 0; c < nch; ++c) {
                const int s = it % NS;
                const uint32_t ph = (it / NS) & 1;
                if (!mbar_wait(&P.empty[s], ph ^ 1, ws.err)) { set_abort(P); break; }
                if (lane == 0) {
                    unsigned char* st = stages + s * kStage;
                    if (dsh) {
                        // 16 rows of the shared down matrix (two 8-row groups of core-matrix tiles),
                        // columns c*dkcs .. +dkcs, then every token's h pieces for those columns
                        const int kc0 = c * dkcs;
                        const uint32_t abytes = dkcs * 16, hbytes = dkcs * 4;
                        P.info[s] = ChunkInfo{total + dt, c, nch, kc0, dkcs};
                        mbar_arrive_expect_tx(&P.full[s], 2 * abytes + n * hbytes);
#pragma unroll
                        for (int q = 0; q < 2; ++q)
                            bulk_load(st + q * abytes, W.sh_down + ((size_t)(dts * 2 + q) * (I / 8) + kc0 / 8) * 64,
                                      abytes, &P.full[s], pol);
                        for (int q = 0; q < n; ++q)
                            bulk_load_plain(st + 2 * abytes + q * hbytes, ws.hb_sh + ((size_t)q * (I / 64) + kc0 / 64) * 128,
                                            hbytes, &P.full[s]);
                    } else {
                        const int e = Rt.uniq[u], s0 = Rt.ustart[u];
                        const int kt0 = c * ck;
                        const int sb0 = dnsb > 1 ? kt0 / 4 : 0, nsbc = dnsb > 1 ? (ck + 3) / 4 : 1;
                        const uint32_t cpb = Q4 ? 1024 : 512;   // code bytes per 32-row step
                        const uint32_t qb = ck * cpb, sb = ck * 128, dbb = nsbc * 128;
                        const uint32_t hb = ck * 256, hsb = ck * 16;
                        P.info[s] = ChunkInfo{total + dt, c, nch, kt0, ck};
                        mbar_arrive_expect_tx(&P.full[s], qb + sb + dbb + ns * (hb + hsb));
                        const size_t qs_stride = Q4 ? W.q4_q_stride : W.q2_q_stride;
                        const uint32_t* scp = Q4 ? W.down_sc4 + (size_t)e * W.q4_sc_stride : W.down_sc + (size_t)e * W.q2_sc_stride;
                        const uint32_t* ddp = Q4 ? W.down_dd4 + (size_t)e * W.q4_dd_stride : W.down_dd + (size_t)e * W.q2_dd_stride;
                        bulk_load(st, W.down_q + (size_t)e * qs_stride + ((size_t)rb * dnkt + kt0) * cpb, qb,
                                  &P.full[s], pol);
                        bulk_load(st + qb, scp + ((size_t)rb * dnkt + kt0) * 32, sb, &P.full[s], pol);
                        bulk_load(st + qb + sb, ddp + ((size_t)rb * dnsb + sb0) * 32, dbb, &P.full[s], pol);
                        unsigned char* hdst = st + qb + sb + dbb;
                        for (int q = 0; q < ns; ++q) {
                            const int slot = Rt.slot[s0 + q];
                            bulk_load_plain(hdst + q * hb, ws.hb_rt + ((size_t)slot * (I / 64) + kt0) * 128, hb,
                                            &P.full[s]);
                            bulk_load_plain(hdst + ns * hb + q * hsb, ws.hsum_rt + (size_t)slot * (I / 16) + 4 * kt0,
                                            hsb, &P.full[s]);
                        }
                    }
                }
                __syncwarp();
                ++it;
            }
            return !aborted(P);
        };
        if constexpr (C::kSplitX) {
            // One token: two streams of gate/up tasks, shared-expert tasks (queue: their numbers, then the
            // down tasks) and routed tasks (queue_rt), taken chunk by chunk in turn, so that a
            // dequantization-bound routed stage and a bandwidth-bound shared-expert stage alternate and every
            // stage's copy is issued two stages ahead of its use.  One shared-expert task leads while the
            // router finishes.  The down tasks follow once both streams are exhausted and this producer's
            // gate/up chunks are all issued (a down task waits only for gate/up tasks that other producers
            // have issued in full or will issue without waiting).  Each queue's next position is in flight
            // while the current task streams.
            int qs = 0, qr = 0;
            int sh_task = -1, sh_c = 0, sh_taken = 0, rt_task = -1, rt_c = 0, dn_pos = 0;
            bool sh_out = false, rt_out = false, pref_rt = false;
            if (lane == 0) qs = (int)atomicAdd(ws.queue, 1u);
            for (;;) {
                if (aborted(P) || refused) break;
                if (!routed && sh_task < 0 && (sh_taken > 0 || sh_out)) {
                    // the router's ids and weights: published by its last CTA through the ready flag (probe
                    // calls route by themselves)
                    if (!ws.probe && !wait_flag(ws.route_ready, ws.err)) { set_abort(P); break; }
                    route();
                    if (lane == 0) qr = (int)atomicAdd(ws.queue_rt, 1u);
                }
                if (sh_task < 0 && !sh_out) {
                    const int q = __shfl_sync(0xffffffffu, qs, 0);
                    if (q < n_sh) {
                        sh_task = q;
                        sh_c = 0;
                        ++sh_taken;
                        if (lane == 0) qs = (int)atomicAdd(ws.queue, 1u);
                    } else {
                        sh_out = true;
                        dn_pos = q;
                    }
                }
                if (routed && rt_task < 0 && !rt_out) {
                    const int q = __shfl_sync(0xffffffffu, qr, 0);
                    if (q < total - n_sh) {
                        rt_task = n_sh + q;
                        rt_c = 0;
                        if (lane == 0) qr = (int)atomicAdd(ws.queue_rt, 1u);
                    } else {
                        rt_out = true;
                    }
                }
                if (sh_task < 0 && rt_task < 0) {
                    if (routed) break;   // both streams exhausted
                    continue;            // the shared stream ran out first: route, then take routed tasks
                }
                const bool use_rt = rt_task >= 0 && (pref_rt || sh_task < 0);
                if (use_rt) {
                    if (!issue_gu(rt_task, rt_c)) break;
                    if (++rt_c == nch_rt) rt_task = -1;
                } else {
                    if (!issue_gu(sh_task, sh_c)) break;
                    if (++sh_c == nch_sh) sh_task = -1;
                }
                pref_rt = !use_rt;
            }
            if (!aborted(P) && !refused && routed) {
                int pos = dn_pos, nxt = 0;
                if (lane == 0) nxt = (int)atomicAdd(ws.queue, 1u);
                for (;;) {
                    const int dt = pos - n_sh;
                    if (dt >= d_total || aborted(P)) break;
                    if (!run_down(dt)) break;
                    pos = __shfl_sync(0xffffffffu, nxt, 0);
                    if (lane == 0) nxt = (int)atomicAdd(ws.queue, 1u);
                }
                asm volatile("" ::"r"(nxt));
            }
            // the prefetched positions are read, so every queue atomic of this CTA has completed before the
            // last CTA resets the queues
            asm volatile("" ::"r"(qs), "r"(qr));
        } else {
            // Two or more tokens: one queue, two ahead (the atomic for the one after next is in flight while
            // this task streams): every shared-expert task (x's int8 pieces replace its bf16 pieces once
            // they are done), then the routed gate/up tasks, then the down tasks.
            int nxt = 0, nxt2 = 0;
            if (lane == 0) {
                nxt = (int)atomicAdd(ws.queue, 1u);
                nxt2 = (int)atomicAdd(ws.queue, 1u);
            }
            for (;;) {
                if (aborted(P) || refused) break;
                const int pos = __shfl_sync(0xffffffffu, nxt, 0);
                if (lane == 0) {
                    nxt = nxt2;
                    nxt2 = (int)atomicAdd(ws.queue, 1u);   // in flight while this task streams
                }
                if (pos >= n_sh && !routed) {
                    if (!ws.probe && !wait_flag(ws.route_ready, ws.err)) { set_abort(P); break; }
                    route();
                }
                if (pos >= total) {
                    const int dt = pos - total;
                    if (dt >= d_total || !run_down(dt)) break;
                    continue;
                }
                const int nch = pos < n_sh ? nch_sh : nch_rt;
                bool ok = true;
                for (int c = 0; c < nch && ok; ++c) ok = issue_gu(pos, c);
                if (!ok) break;
            }
            asm volatile("" ::"r"(nxt), "r"(nxt2));
        }
        producer_finish(P, it, NS, ws.err);
    } else if (warp < CW && !refused) {
        // ------------------------------------------------ consumer warps
        const uint32_t selA = 0x4440u | (uint32_t)t;   // byte t of the index word
        const uint32_t selO = (t >> 1) ? 0xFEDCu : 0xBA98u;   // this lane's group's S word, top bits
        const uint32_t* tselp = tsel + (lane % R);
        const uint32_t* tsgnp = tsgn + (lane % R);
        const uint32_t tb = kAbs ? 0u : smem_addr(tsel);
        const uint32_t hiA = kAbs ? (kTabAddr >> 16) << 16 : 0u;   // bytes 2, 3 of a row's address
        const uint32_t lbA = hiA | ((uint32_t)lane << 2), lbB = hiA | 128u | ((uint32_t)lane << 2);
        const uint32_t selT = 0x7604u | ((uint32_t)t << 4);
        const uint32_t clo = s_cand[0], chi = s_cand[1];
        // B operand lanes: column g of the MMA
        const int jB = g >> 2, pB = g & 3;                // routed: 32-column group, int8 piece
        const uint32_t rot = (5u - 2u * (uint32_t)t) & 31u;   // down: code t of each byte to bits 5..6
        const int jD = g >> 1, pD = g & 1;                    // down, routed B lanes: sub-block, piece
        uint32_t it = 0, cph = 0, ntask = 0;
        bool quantized = false;
        GateUpAcc<NT> A;
        DownAcc<NT> A2;
        int dtcount = 0;
        int tokrow[TPB];
        int tcount = 0;
        for (;;) {
            const int s = it % NS;
            if (!mbar_wait(&P.full[s], (it / NS) & 1, ws.err)) { set_abort(P); break; }
            const ChunkInfo inf = P.info[s];
            if (inf.task < 0 || aborted(P)) break;
            const unsigned char* st = stages + s * kStage;
            const int T_gu = inf.task < n_sh ? n_sh : n_sh + (do_gu ? Rt.nu * rb_per_e : 0);
            if (inf.task >= T_gu) {
                // ---- down projection
            const int dt = inf.task - T_gu;
            const bool dsh = dt >= (do_dn ? Rt.nu * drb : 0);
            if (dsh) {
                if (inf.chunk == 0) {
#pragma unroll
                    for (int tg = 0; tg < DownAcc<NT>::TG; ++tg) A2.sh[tg][0] = A2.sh[tg][1] = A2.sh[tg][2] = A2.sh[tg][3] = 0.f;
                }
                const int kc = inf.cnt;
                const unsigned char* hst = st + 2 * kc * 16;
                for (int ks = warp; ks < kc / 16; ks += CW) {
                    uint2 B[DownAcc<NT>::TG];
#pragma unroll
                    for (int tg = 0; tg < DownAcc<NT>::TG; ++tg) {
                        const int tk = 4 * tg + (g >> 1), p = g & 1;
                        B[tg] = *reinterpret_cast<const uint2*>(
                            tk < n ? hst + (size_t)tk * kc * 4 + ((ks >> 2) * 2 + p) * 128 + ((ks & 3) * 16 + 4 * t) * 2
                                   : zero);
                    }
                    {
                        const unsigned char* base = st + (2 * ks + (t >> 1)) * 128 + g * 16 + (t & 1) * 8;
                        const uint2 r0 = *reinterpret_cast<const uint2*>(base);
                        const uint2 r1 = *reinterpret_cast<const uint2*>(base + kc * 16);
                        const uint32_t Af[4] = {r0.x, r1.x, r0.y, r1.y};
#pragma unroll
                        for (int tg = 0; tg < DownAcc<NT>::TG; ++tg) bmma(A2.sh[tg], Af, B[tg]);
                    }
                }
            } else {
                const int tt = dt, u = tt / drb;
                const int s0 = Rt.ustart[u], ns = Rt.ustart[u + 1] - s0;
                if (inf.chunk == 0) {
                    dtcount = ns;
#pragma unroll
                    for (int q = 0; q < TPB; ++q)
#pragma unroll
                        for (int T = 0; T < 2; ++T) A2.rt[q][T][0] = A2.rt[q][T][1] = 0.f;
                }
                const int ck = inf.cnt;
                const int nsbc = dnsb > 1 ? (ck + 3) / 4 : 1;
                if constexpr (Q4) {
                // codes [ck][32][32 B], scale words [ck][32], (d, dmin) words [nsbc][32], then the slots' h
                // pieces and per-16 sums
                const unsigned char* qv = st;
                const uint32_t* scv = reinterpret_cast<const uint32_t*>(st + ck * 1024);
                const uint32_t* ddv = reinterpret_cast<const uint32_t*>(st + ck * 1152);
                const uint16_t* hst = reinterpret_cast<const uint16_t*>(st + ck * 1152 + nsbc * 128);
                const float* hss = reinterpret_cast<const float*>(st + ck * 1152 + nsbc * 128 + ns * ck * 256);
                const int jj = t >> 1;   // this lane's 16-column group t lies in 32-column sub-block t / 2
                for (int kt = warp; kt < ck; kt += CW) {
                    const int sbi = dnsb > 1 ? ((inf.lo + kt) >> 2) - (inf.lo >> 2) : 0;
                    uint2 Bl[TPB];
                    float S[TPB];
#pragma unroll
                    for (int q = 0; q < TPB; ++q) {
                        Bl[q] = make_uint2(0u, 0u);
                        S[q] = 0.f;
                        if (q < dtcount) {
                            Bl[q] = *reinterpret_cast<const uint2*>(hst + (size_t)q * ck * 128 + (kt * 2 + pD) * 64 + 16 * jD + 4 * t);
                            S[q] = hss[q * ck * 4 + kt * 4 + t];
                        }
                    }
#pragma unroll
                    for (int T = 0; T < 2; ++T) {
                        const int rg = 16 * T + g;
                        const uint2 c0 = *reinterpret_cast<const uint2*>(qv + kt * 1024 + rg * 32 + 8 * t);
                        const uint2 c1 = *reinterpret_cast<const uint2*>(qv + kt * 1024 + (rg + 8) * 32 + 8 * t);
                        uint32_t Af[4][4];
                        q4_down_frags(c0.x, c1.x, Af[0], Af[1]);
                        q4_down_frags(c0.y, c1.y, Af[2], Af[3]);
                        // sum q h = 16 (D - S) over the lane's group; a16 = 16 d sc, mm = dmin m, per row
                        const uint32_t sw0 = scv[kt * 32 + rg], sw1 = scv[kt * 32 + rg + 8];
                        const uint32_t dd0 = ddv[sbi * 32 + rg], dd1 = ddv[sbi * 32 + rg + 8];
                        const float a160 = 16.f * half_bits(dd0 & 0xffffu) * (float)((sw0 >> (8 * jj)) & 0xffu);
                        const float a161 = 16.f * half_bits(dd1 & 0xffffu) * (float)((sw1 >> (8 * jj)) & 0xffu);
                        const float mm0 = half_bits(dd0 >> 16) * (float)((sw0 >> (16 + 8 * jj)) & 0xffu);
                        const float mm1 = half_bits(dd1 >> 16) * (float)((sw1 >> (16 + 8 * jj)) & 0xffu);
#pragma unroll
                        for (int q = 0; q < TPB; ++q) {
                            float Dv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                            for (int j = 0; j < 4; ++j) bmma(Dv, Af[j], jD == j ? Bl[q] : make_uint2(0u, 0u));
                            A2.rt[q][T][0] = fmaf(a160, (Dv[0] + Dv[1]) - S[q], A2.rt[q][T][0]);
                            A2.rt[q][T][0] = fmaf(-mm0, S[q], A2.rt[q][T][0]);
                            A2.rt[q][T][1] = fmaf(a161, (Dv[2] + Dv[3]) - S[q], A2.rt[q][T][1]);
                            A2.rt[q][T][1] = fmaf(-mm1, S[q], A2.rt[q][T][1]);
                        }
                    }
                }
                } else {
                const unsigned char* qv = st;
                const uint32_t* scv = reinterpret_cast<const uint32_t*>(st + ck * 512);
                const uint32_t* ddv = reinterpret_cast<const uint32_t*>(st + ck * 640);
                const uint16_t* hst = reinterpret_cast<const uint16_t*>(st + ck * 640 + nsbc * 128);
                const float* hss = reinterpret_cast<const float*>(st + ck * 640 + nsbc * 128 + ns * ck * 256);
                for (int kt = warp; kt < ck; kt += CW) {
                    const int sbi = dnsb > 1 ? ((inf.lo + kt) >> 2) - (inf.lo >> 2) : 0;   // superblock in the stage
                    uint2 Bl[TPB];
                    float S[TPB];
#pragma unroll
                    for (int q = 0; q < TPB; ++q) {
                        Bl[q] = make_uint2(0u, 0u);
                        S[q] = 0.f;
                        if (q < dtcount) {
                            Bl[q] = *reinterpret_cast<const uint2*>(hst + (size_t)q * ck * 128 + (kt * 2 + pD) * 64 + 16 * jD + 4 * t);
                            S[q] = hss[q * ck * 4 + kt * 4 + t];
                        }
                    }
#pragma unroll
                    for (int T = 0; T < 2; ++T) {
                        const int rg = 16 * T + g;
                        const uint4 q0 = *reinterpret_cast<const uint4*>(qv + kt * 512 + rg * 16);
                        const uint4 q1 = *reinterpret_cast<const uint4*>(qv + kt * 512 + (rg + 8) * 16);
                        const uint32_t w0[4] = {q0.x, q0.y, q0.z, q0.w}, w1[4] = {q1.x, q1.y, q1.z, q1.w};
                        uint32_t Af[4][4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t y0 = (__funnelshift_l(w0[j], w0[j], rot) & 0x60606060u) | 0x80808080u;
                            const uint32_t y1 = (__funnelshift_l(w1[j], w1[j], rot) & 0x60606060u) | 0x80808080u;
                            Af[j][0] = __byte_perm(y0, 0x3f3f3f3fu, 0x5140);
                            Af[j][1] = __byte_perm(y1, 0x3f3f3f3fu, 0x5140);
                            Af[j][2] = __byte_perm(y0, 0x3f3f3f3fu, 0x7362);
                            Af[j][3] = __byte_perm(y1, 0x3f3f3f3fu, 0x7362);
                        }
                        // this lane's sub-block t: a4 = 4 d sc, mm = dmin m, per row
                        const uint32_t sw0 = scv[kt * 32 + rg], sw1 = scv[kt * 32 + rg + 8];
                        const uint32_t dd0 = ddv[sbi * 32 + rg], dd1 = ddv[sbi * 32 + rg + 8];
                        const float d0 = half_bits(dd0 & 0xffffu), m0 = half_bits(dd0 >> 16);
                        const float d1 = half_bits(dd1 & 0xffffu), m1 = half_bits(dd1 >> 16);
                        const uint32_t b0 = sw0 >> (8 * t), b1 = sw1 >> (8 * t);
                        const float a40 = fmaf(__uint_as_float(0x4b000000u | (b0 & 15u)), 4.f * d0, -33554432.f * d0);
                        const float a41 = fmaf(__uint_as_float(0x4b000000u | (b1 & 15u)), 4.f * d1, -33554432.f * d1);
                        const float mm0 = fmaf(__uint_as_float(0x4b000000u | ((b0 >> 4) & 15u)), m0, -8388608.f * m0);
                        const float mm1 = fmaf(__uint_as_float(0x4b000000u | ((b1 >> 4) & 15u)), m1, -8388608.f * m1);
                        // no branch on the entry's slot count: an absent slot's h and S are zero
#pragma unroll
                        for (int q = 0; q < TPB; ++q) {
                            float Dv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                            for (int j = 0; j < 4; ++j) bmma(Dv, Af[j], jD == j ? Bl[q] : make_uint2(0u, 0u));
                            A2.rt[q][T][0] = fmaf(a40, (Dv[0] + Dv[1]) - S[q], A2.rt[q][T][0]);
                            A2.rt[q][T][0] = fmaf(-mm0, S[q], A2.rt[q][T][0]);
                            A2.rt[q][T][1] = fmaf(a41, (Dv[2] + Dv[3]) - S[q], A2.rt[q][T][1]);
                            A2.rt[q][T][1] = fmaf(-mm1, S[q], A2.rt[q][T][1]);
                        }
                    }
                }
                }
            }
                __syncwarp();
                if (lane == 0) mbar_arrive(&P.empty[s]);
            if (inf.chunk == inf.nchunk - 1) {
                // task end: this warp's partials into the task's reduction buffer (the epilogue warp
                // finishes the task)
                const int b = (int)(ntask % C::NB);
                if (!ring_acquire(RR, b, (int)(ntask / C::NB), ws.err)) { set_abort(P); break; }
                float* rbuf = red + (size_t)b * CW * C::kRedPer + warp * C::kRedPer;
                if (dsh) {
                    // this lane's token is 4 tg + t (its columns 2t, 2t+1 are that token's two pieces)
#pragma unroll
                    for (int tg = 0; tg < DownAcc<NT>::TG; ++tg) {
                        if (4 * tg + t < n) {
                            rbuf[(4 * tg + t) * 16 + g] = A2.sh[tg][0] + A2.sh[tg][1];
                            rbuf[(4 * tg + t) * 16 + g + 8] = A2.sh[tg][2] + A2.sh[tg][3];
                        }
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < TPB; ++q) {
#pragma unroll
                        for (int T = 0; T < 2; ++T) {
#pragma unroll
                            for (int r = 0; r < 2; ++r) {
                                float v = A2.rt[q][T][r];
                                v += __shfl_xor_sync(0xffffffffu, v, 1);
                                v += __shfl_xor_sync(0xffffffffu, v, 2);
                                if (t == 0) rbuf[q * 32 + 16 * T + g + 8 * r] = v;
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) ring_publish(RR, b, inf.task);
                ++ntask;
            }
                ++it;
                continue;
            }
            // ---- gate and up projections
            const bool sh = inf.task < n_sh;
            if (!C::kSplitX && !sh && !quantized) {
                // first routed stage: every consumer warp is done with the shared tasks' bf16 pieces;
                // x becomes four int8 pieces per token in the same buffer
                if (!cons_sync(P, cph, ws.err)) break;
                quantize_x(x, D.act_bf16, n, H, s_f, xq, tid, CW * 32);
                quantized = true;
                if (!cons_sync(P, cph, ws.err)) break;
            }
            if (sh) {
                if (inf.chunk == 0) {
#pragma unroll
                    for (int tg = 0; tg < GateUpAcc<NT>::TG; ++tg)
#pragma unroll
                        for (int T = 0; T < 2; ++T) A.sh[tg][T][0] = A.sh[tg][T][1] = A.sh[tg][T][2] = A.sh[tg][T][3] = 0.f;
                }
                const int kc = inf.cnt;                                 // columns of the chunk
                const uint16_t* xb = reinterpret_cast<const uint16_t*>(xbuf);
                for (int ks = warp; ks < kc / 16; ks += CW) {
                    const int col = inf.lo + 16 * ks;
                    uint2 B[GateUpAcc<NT>::TG];
#pragma unroll
                    for (int tg = 0; tg < GateUpAcc<NT>::TG; ++tg) {
                        const int tk = 4 * tg + (g >> 1), p = g & 1;
                        B[tg] = *reinterpret_cast<const uint2*>(
                            tk < n ? reinterpret_cast<const unsigned char*>(xb + (size_t)(tk * 2 + p) * H + col + 4 * t)
                                   : zero);
                    }
#pragma unroll
                    for (int T = 0; T < 2; ++T) {   // gate, up: 8 rows each (the MMA's rows g + 8 repeat rows g)
                        const uint2 r0 = *reinterpret_cast<const uint2*>(st + T * (kc * 16) + (2 * ks + (t >> 1)) * 128 +
                                                                         g * 16 + (t & 1) * 8);
                        const uint32_t Af[4] = {r0.x, r0.x, r0.y, r0.y};
#pragma unroll
                        for (int tg = 0; tg < GateUpAcc<NT>::TG; ++tg) bmma(A.sh[tg][T], Af, B[tg]);
                    }
                }
            } else {
                const int tt = inf.task - n_sh, u = tt / rb_per_e;
                const int s0 = Rt.ustart[u], ns = Rt.ustart[u + 1] - s0;
                if (inf.chunk == 0) {
                    tcount = ns;
#pragma unroll
                    for (int q = 0; q < TPB; ++q) {
                        tokrow[q] = q < ns ? Rt.slot[s0 + q] / k : 0;
#pragma unroll
                        for (int T = 0; T < 4; ++T) A.rt[q][T][0] = A.rt[q][T][1] = 0.f;
                    }
                }
                const int ck = inf.cnt;
                if constexpr (Q4) {
                    // gate codes, up codes [ck][32][32 B], scale words [2][ck][32], (d, dmin) words [2][ck/4][32]
                    const uint32_t* scw = reinterpret_cast<const uint32_t*>(st + 2 * ck * 1024);
                    const uint32_t* ddw = scw + 2 * ck * 32;
                    const int jj = t >> 1;            // this lane's 32-column half of a step
                    const int p0 = 2 * (t & 1);       // and its two int8 pieces
                    for (int kt = warp; kt < ck; kt += CW) {
                        const int col = 64 * (inf.lo + kt);
                        uint2 B[TPB][2];
                        float xs[TPB];
#pragma unroll
                        for (int q = 0; q < TPB; ++q) {
                            const unsigned char* live =
                                xq + (size_t)(tokrow[q] * 4 + pB) * H + col + 32 * jB + 8 * t;
                            B[q][0] = *reinterpret_cast<const uint2*>(q < tcount && jB == 0 ? live : zero);
                            B[q][1] = *reinterpret_cast<const uint2*>(q < tcount && jB == 1 ? live : zero);
                            // the min term of the lane's half, once per half (even t)
                            xs[q] = q < tcount && (t & 1) == 0 ? xsum[tokrow[q] * (H / 32) + (col >> 5) + jj] : 0.f;
                        }
#pragma unroll
                        for (int T = 0; T < 4; ++T) {
                            const int mt = T >> 1, rg = 16 * (T & 1) + g;
                            const unsigned char* pay = st + (mt * ck + kt) * 1024 + rg * 32 + 8 * t;
                            const uint2 c0 = *reinterpret_cast<const uint2*>(pay);
                            const uint2 c1 = *reinterpret_cast<const uint2*>(pay + 256);   // row rg + 8
                            constexpr uint32_t M = 0x0F0F0F0Fu;
                            const uint32_t A0[4] = {c0.x & M, c1.x & M, (c0.x >> 4) & M, (c1.x >> 4) & M};
                            const uint32_t A1[4] = {c0.y & M, c1.y & M, (c0.y >> 4) & M, (c1.y >> 4) & M};
                            const uint32_t sw0 = scw[(mt * ck + kt) * 32 + rg], sw1 = scw[(mt * ck + kt) * 32 + rg + 8];
                            const uint32_t dw0 = ddw[(mt * (ck / 4) + kt / 4) * 32 + rg];
                            const uint32_t dw1 = ddw[(mt * (ck / 4) + kt / 4) * 32 + rg + 8];
                            const float a0 = half_bits(dw0 & 0xffffu) * (float)((sw0 >> (8 * jj)) & 0xffu);
                            const float a1 = half_bits(dw1 & 0xffffu) * (float)((sw1 >> (8 * jj)) & 0xffu);
                            const float m0 = half_bits(dw0 >> 16) * (float)((sw0 >> (16 + 8 * jj)) & 0xffu);
                            const float m1 = half_bits(dw1 >> 16) * (float)((sw1 >> (16 + 8 * jj)) & 0xffu);
#pragma unroll
                            for (int q = 0; q < TPB; ++q) {   // absent tokens: B = 0, xs = 0
                                int Dv[4];
                                imma_z(Dv, A0, B[q][0]);
                                imma(Dv, A1, B[q][1]);
                                const float c0f = s_cs[tokrow[q]][p0], c1f = s_cs[tokrow[q]][p0 + 1];
                                A.rt[q][T][0] = fmaf(a0, fmaf((float)Dv[0], c0f, (float)Dv[1] * c1f), A.rt[q][T][0]);
                                A.rt[q][T][0] = fmaf(-m0, xs[q], A.rt[q][T][0]);
                                A.rt[q][T][1] = fmaf(a1, fmaf((float)Dv[2], c0f, (float)Dv[3] * c1f), A.rt[q][T][1]);
                                A.rt[q][T][1] = fmaf(-m1, xs[q], A.rt[q][T][1]);
                            }
                        }
                    }
                } else {
                const int kpw = ck >= CW ? ck / CW : 1;
                const int kb = warp * kpw;
                if (kb < ck) {
                    int ai[TPB][4][4];
#pragma unroll
                    for (int q = 0; q < TPB; ++q)
#pragma unroll
                        for (int T = 0; T < 4; ++T) ai[q][T][0] = ai[q][T][1] = ai[q][T][2] = ai[q][T][3] = 0;
                    for (int kq = 0; kq < kpw; ++kq) {
                        const int kt = kb + kq;
                        const int col = 64 * (inf.lo + kt);
                        uint2 B[TPB][2];
#pragma unroll
                        for (int q = 0; q < TPB; ++q) {
                            const unsigned char* live =
                                xq + (size_t)(tokrow[q] * 4 + pB) * H + col + 32 * jB + 8 * t;
                            B[q][0] = *reinterpret_cast<const uint2*>(q < tcount && jB == 0 ? live : zero);
                            B[q][1] = *reinterpret_cast<const uint2*>(q < tcount && jB == 1 ? live : zero);
                        }
#pragma unroll
                        for (int T = 0; T < 4; ++T) {
                            const unsigned char* pay = st + (T >> 1) * (ck * 512) + kt * 512 + (16 * (T & 1) + g) * 16;
                            const uint4 r0 = *reinterpret_cast<const uint4*>(pay);
                            const uint4 r1 = *reinterpret_cast<const uint4*>(pay + 128);
                            uint32_t A0[4], A1[4];
                            if (C::kRows) {
                                iq2_chunk_rows(r0.x, r0.y, tb, lbA, lbB, selT, clo, chi, A0[0], A0[2]);
                                iq2_chunk_rows(r1.x, r1.y, tb, lbA, lbB, selT, clo, chi, A0[1], A0[3]);
                                iq2_chunk_rows(r0.z, r0.w, tb, lbA, lbB, selT, clo, chi, A1[0], A1[2]);
                                iq2_chunk_rows(r1.z, r1.w, tb, lbA, lbB, selT, clo, chi, A1[1], A1[3]);
                            } else {
                                iq2_chunk_s8<R>(r0.x, r0.y, selA, 8 * t, tselp, tsgnp, clo, chi, A0[0], A0[2]);
                                iq2_chunk_s8<R>(r1.x, r1.y, selA, 8 * t, tselp, tsgnp, clo, chi, A0[1], A0[3]);
                                iq2_chunk_s8<R>(r0.z, r0.w, selA, 8 * t, tselp, tsgnp, clo, chi, A1[0], A1[2]);
                                iq2_chunk_s8<R>(r1.z, r1.w, selA, 8 * t, tselp, tsgnp, clo, chi, A1[1], A1[3]);
                            }
                            const int o0 = iq2_odd(r0.y, r0.w, selO);
                            const int o1 = iq2_odd(r1.y, r1.w, selO);
                            // no branch on the entry's token count: an absent token's B is zero
#pragma unroll
                            for (int q = 0; q < TPB; ++q) {
                                int Dv[4];
                                imma_z(Dv, A0, B[q][0]);
                                imma(Dv, A1, B[q][1]);
                                ai[q][T][0] += Dv[0] * o0;
                                ai[q][T][1] += Dv[1] * o0;
                                ai[q][T][2] += Dv[2] * o1;
                                ai[q][T][3] += Dv[3] * o1;
                            }
                        }
                    }
                    // one superblock: x d/8 and the columns' piece scales
                    const uint16_t* dq = reinterpret_cast<const uint16_t*>(st + 2 * ck * 512);
                    const int sbl = kb / 4;
                    const int p0 = 2 * (t & 1);
#pragma unroll
                    for (int T = 0; T < 4; ++T) {
                        const uint16_t* dm = dq + (T >> 1) * (ck / 4) * 32 + sbl * 32 + 16 * (T & 1) + g;
                        const float d0 = half_bits(dm[0]) * 0.125f, d1 = half_bits(dm[8]) * 0.125f;
#pragma unroll
                        for (int q = 0; q < TPB; ++q) {   // absent tokens: ai = 0
                            const float c0 = s_cs[tokrow[q]][p0], c1 = s_cs[tokrow[q]][p0 + 1];
                            A.rt[q][T][0] = fmaf((float)ai[q][T][0], d0 * c0, A.rt[q][T][0]);
                            A.rt[q][T][0] = fmaf((float)ai[q][T][1], d0 * c1, A.rt[q][T][0]);
                            A.rt[q][T][1] = fmaf((float)ai[q][T][2], d1 * c0, A.rt[q][T][1]);
                            A.rt[q][T][1] = fmaf((float)ai[q][T][3], d1 * c1, A.rt[q][T][1]);
                        }
                    }
                }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&P.empty[s]);
            if (inf.chunk == inf.nchunk - 1) {
                // task end: this warp's partials into the task's reduction buffer (the epilogue warp
                // finishes the task)
                const int b = (int)(ntask % C::NB);
                if (!ring_acquire(RR, b, (int)(ntask / C::NB), ws.err)) { set_abort(P); break; }
                float* rbuf = red + (size_t)b * CW * C::kRedPer + warp * C::kRedPer;
                if (sh) {
                    // this lane's token is 4 tg + t: its columns 2t, 2t+1 are that token's two pieces
#pragma unroll
                    for (int tg = 0; tg < GateUpAcc<NT>::TG; ++tg)
#pragma unroll
                        for (int T = 0; T < 2; ++T)
                            if (4 * tg + t < n) rbuf[(4 * tg + t) * 16 + T * 8 + g] = A.sh[tg][T][0] + A.sh[tg][T][1];
                } else {
#pragma unroll
                    for (int q = 0; q < TPB; ++q) {
#pragma unroll
                        for (int T = 0; T < 4; ++T) {
#pragma unroll
                            for (int r = 0; r < 2; ++r) {
                                float v = A.rt[q][T][r];
                                v += __shfl_xor_sync(0xffffffffu, v, 1);
                                v += __shfl_xor_sync(0xffffffffu, v, 2);
                                if (t == 0) rbuf[q * 64 + (T >> 1) * 32 + 16 * (T & 1) + g + 8 * r] = v;
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) ring_publish(RR, b, inf.task);
                ++ntask;
            }
            ++it;
        }
        if (lane == 0) ring_exit(RR, (int)ntask);
    } else if (warp == CW + 1 && !refused) {
        // ------------------------------------------------ epilogue warp
        for (uint32_t j = 0; ring_take(RR, j, C::NB, CW, ws.err); ++j) {
            const int b = (int)(j % C::NB);
            const float* rbuf = red + (size_t)b * CW * C::kRedPer;
            const int task = RR.task[b];
            const int T_gu = task < n_sh ? n_sh : n_sh + (do_gu ? Rt.nu * rb_per_e : 0);
            if (task >= T_gu) {
                // ---- down projection: y of the task's rows
                const int dt = task - T_gu;
            const int nd_rt = do_dn ? Rt.nu * drb : 0;
            if (dt >= nd_rt) {
                for (int q = lane; q < 16 * n; q += 32) {   // (token, row) pairs
                    const int tok = q >> 4, row = q & 15;
                    float y = 0.f;
                    for (int w = 0; w < CW; ++w) y += rbuf[w * C::kRedPer + tok * 16 + row];
                    (ws.probe ? ws.probe_out : ws.y_sh)[(size_t)tok * H + 16 * (dt - nd_rt) + row] = y;
                }
            } else {
                const int tt = dt, u = tt / drb, rb = tt % drb;
                const int s0 = Rt.ustart[u], ns = Rt.ustart[u + 1] - s0;
                for (int q = 0; q < ns; ++q) {
                    float y = 0.f;
                    for (int w = 0; w < CW; ++w) y += rbuf[w * C::kRedPer + q * 32 + lane];
                    const int slot = Rt.slot[s0 + q];
                    if (ws.probe) ws.probe_out[(size_t)(slot / k) * H + 32 * rb + lane] = y;
                    else ws.y_rt[(size_t)slot * H + 32 * rb + lane] = y;
                }
            }
                ring_free(RR, j, C::NB);
                continue;
            }
            const bool sh = task < n_sh;
            if (sh) {
                for (int q = lane; q < 8 * n; q += 32) {   // (token, row) pairs
                    const int tok = q >> 3, row = q & 7;
                    float gv = 0.f, uv = 0.f;
                    for (int w = 0; w < CW; ++w) {
                        gv += rbuf[w * C::kRedPer + tok * 16 + row];
                        uv += rbuf[w * C::kRedPer + tok * 16 + 8 + row];
                    }
                    const int c = 8 * task + row;
                    if (ws.probe) {
                        ws.probe_out[(size_t)tok * 2 * I + c] = gv;
                        ws.probe_out[(size_t)tok * 2 * I + I + c] = uv;
                    } else {
                        const float h = silu(gv) * uv;
                        const uint32_t hi = bf16_bits(h);
                        const uint32_t lo = bf16_bits(h - __uint_as_float(hi << 16));
                        uint16_t* hb = ws.hb_sh + (size_t)tok * 2 * I;
                        hb[hsh_index(c, 0)] = (uint16_t)hi;
                        hb[hsh_index(c, 1)] = (uint16_t)lo;
                    }
                }
            } else {
                const int tt = task - n_sh, u = tt / rb_per_e, rb = tt % rb_per_e;
                const int s0 = Rt.ustart[u], ns = Rt.ustart[u + 1] - s0;
                for (int q = 0; q < ns; ++q) {
                    const int row = lane;
                    float gv = 0.f, uv = 0.f;
                    for (int w = 0; w < CW; ++w) {
                        gv += rbuf[w * C::kRedPer + q * 64 + row];
                        uv += rbuf[w * C::kRedPer + q * 64 + 32 + row];
                    }
                    const int slot = Rt.slot[s0 + q];
                    const int c = 32 * rb + row;
                    if (ws.probe) {
                        ws.probe_out[(size_t)(slot / k) * 2 * I + c] = gv;
                        ws.probe_out[(size_t)(slot / k) * 2 * I + I + c] = uv;
                    } else {
                        const float h = silu(gv) * uv;
                        const uint32_t hi = bf16_bits(h);
                        const float hf = __uint_as_float(hi << 16);
                        const uint32_t lo = bf16_bits(h - hf);
                        uint16_t* hb = ws.hb_rt + (size_t)slot * 2 * I;
                        hb[hrt_index(c, 0)] = (uint16_t)hi;
                        hb[hrt_index(c, 1)] = (uint16_t)lo;
                        float hs = hf + __uint_as_float(lo << 16);
#pragma unroll
                        for (int m = 1; m <= 8; m <<= 1) hs += __shfl_xor_sync(0xffffffffu, hs, m);
                        if ((lane & 15) == 0) ws.hsum_rt[(size_t)slot * (I / 16) + 2 * rb + (lane >> 4)] = hs;
                    }
                }
            }
            if (!ws.probe) {
                // h of this task is complete: publish it to the down tasks (the warp barrier orders every
                // lane's stores before lane 0's fence, which is cumulative)
                __syncwarp();
                if (lane == 0) {
                    __threadfence();
                    atomicAdd(ws.gu_done + (sh ? 0 : 1 + (task - n_sh) / rb_per_e), 1u);
                }
            }
            ring_free(RR, j, C::NB);
        }
    }
    griddep_launch();
    // last CTA to leave resets the task queue for the next forward
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        s_last = atomicAdd(ws.done, 1u) == gridDim.x - 1;
        if (s_last) {
            *ws.queue = 0;
            *ws.queue_rt = 0;
            *ws.done = 0;
            *ws.route_ready = 0;
        }
    }
    // the last CTA also clears the gate/up completion counters for the next forward
    __syncthreads();
    if (s_last && !ws.probe) {
        for (int i = tid; i < 1 + kMaxSlots; i += blockDim.x) ws.gu_done[i] = 0;
        if (tid == 0 && ws.chain_wait) *ws.chain_wait = 0;
    }
}

// ---------------------------------------------------------------- combine
// out[t][r] = y_shared[t][r] + sum_j w[t][j] y[t*k + j][r], j in rank order
// (then x[t][r] + that, when the call asks for the residual).
// Chained layers: once every thread of the CTA has written its part of out,
// one thread publishes it (fence, then count) to the next layer.
__device__ __forceinline__ void chain_count(uint32_t* chain_done) {
    if (!chain_done) return;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(chain_done, 1u);
    }
}

// out[i] (token t = i / H, row r = i % H).
__device__ __forceinline__ void combine_one(const Dims& D, const DecodeWs& ws, float* out, int64_t i) {
    const int H = D.H, k = D.k;
    const int t = (int)(i / H), r = (int)(i % H);
    float w[16], y[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {   // all loads first: k <= 16
        if (j < k) {
            w[j] = __ldcg(ws.wts + t * k + j);
            y[j] = __ldcg(ws.y_rt + (int64_t)(t * k + j) * H + r);
        }
    }
    float acc = D.has_shared ? __ldcg(ws.y_sh + (int64_t)t * H + r) : 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if (j < k) acc = fmaf(w[j], y[j], acc);
    out[i] = ws.xres ? act_at(ws.xres, i, D.act_bf16) + acc : acc;
}

__global__ void __launch_bounds__(256) k_combine_decode(Dims D, DecodeWs ws, float* out, int n) {
    griddep_launch();   // chained layers: the next layer's router may load its rows now
    griddep_wait();     // y of the projection grid
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // the projection grid refused the grid: out stays as it was
    if (i < (int64_t)n * D.H && !__ldcg(ws.grid_refused)) combine_one(D, ws, out, i);
    chain_count(ws.chain_done);
}

// The combine with directional steering of the layer output: one CTA per
// token; y = y_shared + sum_j w_j y_j as above, then y - F v (v . y) with
// v . y summed in a fixed order (per thread over its columns, then the CTA),
// one FMA per element, then x + that when the call asks for the residual.
constexpr int kSteerThreads = 1024;   // few tokens: one wide CTA per token
constexpr int kSteerCols = 4;          // columns per thread (H <= 4096)

// One token (the CTA's) of the steered combine.
__device__ __forceinline__ void steer_one(const Dims& D, const DecodeWs& ws, float* out) {
    __shared__ float red[kSteerThreads / 32];
    const int t = blockIdx.x, H = D.H, k = D.k;
    float acc[kSteerCols];
    float dot = 0.f;
#pragma unroll
    for (int q = 0; q < kSteerCols; ++q) {
        const int r = threadIdx.x + q * kSteerThreads;
        if (r < H) {
            float a = D.has_shared ? __ldcg(ws.y_sh + (int64_t)t * H + r) : 0.f;
            for (int j = 0; j < k; ++j)
                a = fmaf(__ldcg(ws.wts + t * k + j), __ldcg(ws.y_rt + (int64_t)(t * k + j) * H + r), a);
            acc[q] = a;
            dot = fmaf(ws.steer_v[r], a, dot);
        }
    }
    const float sF = ws.steer_F * cta_sum_fixed<kSteerThreads>(dot, red);
#pragma unroll
    for (int q = 0; q < kSteerCols; ++q) {
        const int r = threadIdx.x + q * kSteerThreads;
        if (r < H) {
            const float y = fmaf(-sF, ws.steer_v[r], acc[q]);
            out[(int64_t)t * H + r] = ws.xres ? act_at(ws.xres, (int64_t)t * H + r, D.act_bf16) + y : y;
        }
    }
}

__global__ void __launch_bounds__(kSteerThreads) k_combine_steer_decode(Dims D, DecodeWs ws, float* out, int n) {
    griddep_launch();   // chained layers: the next layer's router may load its rows now
    griddep_wait();     // y of the projection grid
    // the projection grid refused the grid: out stays as it was (a CTA-uniform test)
    if (!__ldcg(ws.grid_refused)) steer_one(D, ws, out);
    chain_count(ws.chain_done);
}

// ---------------------------------------------------------------- caller routing
__global__ void k_routing_in(const int32_t* ids_in, const float* wts_in, int nslots, int E, int32_t* ids, float* wts,
                             uint32_t* ready, uint32_t* err) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nslots; i += gridDim.x * blockDim.x) {
        const int e = ids_in[i];
        const bool ok = e >= 0 && e < E;
        if (!ok) set_err(err, kErrBounds);
        ids[i] = ok ? e : 0;
        wts[i] = ok ? wts_in[i] : 0.f;
    }
    if (ready) {
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(ready), "r"(1u) : "memory");
        }
    }
}

// Expert-parallel combine: out[t][r] = base[t][r] + sum_j w[t][j] y[t k + j][r], j ascending, one FMA
// per slot (the order of the layer's own combine); base may be absent (zero).
__global__ void __launch_bounds__(256) k_combine_slots(const float* y, const float* w, const float* base, int n, int k,
                                                       int H, float* out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)n * H) return;
    const int t = (int)(i / H), r = (int)(i % H);
    float acc = base ? base[i] : 0.f;
    for (int j = 0; j < k; ++j) acc = fmaf(w[t * k + j], y[(int64_t)(t * k + j) * H + r], acc);
    out[i] = acc;
}

cudaError_t launch_combine_slots(const float* y, const float* w, const float* base, int n, int k, int H, float* out,
                                 cudaStream_t st) {
    const int64_t nel = (int64_t)n * H;
    k_combine_slots<<<(unsigned)((nel + 255) / 256), 256, 0, st>>>(y, w, base, n, k, H, out);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- grid tables
// The decode plan's tables of a grid, made once when the grid is loaded (one
// CTA of 256 threads): the distinct magnitudes in ascending order are classes
// 0..3; gtab[a] holds the classes of row a's eight elements as nibbles,
// gtab[256 + sg] the sign flags of the 7-bit sign field sg as bit 2 of each
// nibble (element 7 negative for odd popcount), gtab[384..387] the magnitudes
// as int8 bytes, their negatives, whether the grid is refused (more than four
// distinct values, or a value above 127) and the number of distinct values.
__global__ void __launch_bounds__(256) k_grid_tables(const uint8_t* grid, uint32_t* gtab, uint32_t* rows) {
    __shared__ int cls[256];
    __shared__ uint32_t words[384];
    const int tid = threadIdx.x;
    cls[tid] = 0;
    __syncthreads();
    for (int q = tid; q < 2048; q += 256) cls[grid[q]] = 1;
    __syncthreads();
    if (tid == 0) {
        int nv = 0;
        uint32_t lo = 0, hi = 0;
        bool big = false;
        for (int v = 0; v < 256; ++v) {
            if (!cls[v]) continue;
            if (nv < 4) {
                lo |= (uint32_t)v << (8 * nv);
                hi |= (uint32_t)((-v) & 0xff) << (8 * nv);
            }
            big |= v > 127;
            cls[v] = 1 + (nv < 4 ? nv : 3);
            ++nv;
        }
        gtab[384] = lo;
        gtab[385] = hi;
        gtab[386] = (nv > 4 || big) ? 1u : 0u;
        gtab[387] = (uint32_t)nv;
    }
    __syncthreads();
    uint32_t w = 0;
    for (int i = 0; i < 8; ++i) w |= (uint32_t)(cls[grid[tid * 8 + i]] - 1) << (4 * i);
    gtab[tid] = w;
    words[tid] = w;
    if (tid < 128) {
        uint32_t sgw = ((uint32_t)__popc(tid) & 1u) << 30;
        for (int i = 0; i < 7; ++i) sgw |= ((uint32_t)(tid >> i) & 1u) << (4 * i + 2);
        gtab[256 + tid] = sgw;
        words[256 + tid] = sgw;
    }
    __syncthreads();
    // rows form: one copy of the row's class word per lane, then one of its sign word
    for (int i = tid; i < 256 * 64; i += 256) {
        const int r = i >> 6;
        rows[i] = words[(i & 32) ? 256 + (r & 127) : r];
    }
}

cudaError_t launch_grid_tables(const uint8_t* grid, uint32_t* gtab, uint32_t* rows, cudaStream_t st) {
    k_grid_tables<<<1, 256, 0, st>>>(grid, gtab, rows);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- failure-path check
// One warp waits, with the kernels' bounded wait routine, on an mbarrier that
// no thread ever arrives at: the wait gives up after kWaitNs, records
// kErrTimeout in the error word and the kernel returns.
__global__ void k_wait_selftest(uint32_t* err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    mbar_wait(&bar, 0, err);
}

cudaError_t launch_wait_selftest(uint32_t* err, cudaStream_t st) {
    k_wait_selftest<<<1, 32, 0, st>>>(err);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- launchers
template <int NT, bool Q4>
size_t gateup_smem_bytes_t(const Dims& D, int n) {
    using C = GateUpCfg<NT, Q4>;
    if (!Q4 && C::kRows)   // up to the table's end, less the static shared memory (at least 4 KB) before it
        return (size_t)kTabAddr + 256 * 64 * 4 + (size_t)(C::kSplitX ? 2 : 1) * n * D.H * 4 + 64 - 4096;
    return (size_t)C::NS * C::kStage + 4 * ((size_t)(Q4 ? 0 : C::kTabWords) + C::kRedFloats) +
           (size_t)(C::kSplitX ? 2 : 1) * n * D.H * 4 + 64 + (Q4 ? (size_t)n * (D.H / 32) * 4 : 0);
}
template <int NT>
size_t gateup_smem_bytes(const Dims& D, int n) {
    return D.q4 ? gateup_smem_bytes_t<NT, true>(D, n) : gateup_smem_bytes_t<NT, false>(D, n);
}

size_t router_smem_bytes(const Dims& D, int n) {
    return (size_t)kRE * D.H * 4 + (size_t)n * D.H * (D.act_bf16 ? 2 : 4);
}

// Events (optional): ev[2i] / ev[2i+1] recorded around launch i.  Under
// stream capture they become external event-record nodes, so that replays
// of the graph time each kernel.
struct Marks {
    cudaEvent_t const* ev;
    cudaStream_t st;
    int i = 0;
    unsigned flags = 0;
    Marks(cudaEvent_t const* e, cudaStream_t s) : ev(e), st(s) {
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

const char* const kDecodeKernels[3] = {"k_router_decode", "k_moe_decode", "k_combine_decode"};


// Dynamic shared memory opt-in: raised once per (kernel, device) to the
// device's per-block maximum, outside any stream capture (the first forward
// of a shape does it).
template <typename K>
cudaError_t configure(K kernel) {
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, bool> done;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
    if (done.count(key)) return cudaSuccess;
    int optin = 0;
    err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (err != cudaSuccess) return err;
    cudaFuncAttributes fa;
    err = cudaFuncGetAttributes(&fa, kernel);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes);
    if (err != cudaSuccess) return err;
    done[key] = true;
    return cudaSuccess;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int NT, bool Q4>
cudaError_t launch_decode_t(const Weights& W, const Dims& D, const DecodeWs& ws, const void* x, int n, float* out,
                            int n_sm, cudaStream_t st, cudaEvent_t const* ev, const int32_t* ids_in,
                            const float* wts_in) {
    cudaError_t err;
    const size_t s1 = gateup_smem_bytes<NT>(D, n);
    if ((err = configure(k_moe_decode<NT, Q4>)) != cudaSuccess) return err;
    if ((err = configure(k_router_decode<NT>)) != cudaSuccess) return err;
    Marks mk(ev, st);
    const bool pdl = ev == nullptr;   // profiled runs keep the kernels apart
    const int rgrid = (D.E + kRE - 1) / kRE;
    mk.before();
    if (ids_in) {   // caller routing: copied (and checked) in place of the router's, then published
        k_routing_in<<<1, 128, 0, st>>>(ids_in, wts_in, n * D.k, D.E, ws.ids, ws.wts, ws.route_ready, ws.err);
        err = cudaGetLastError();
    } else {
        // chained layers: a programmatic dependent of the previous layer's combine (it loads its rows, then waits)
        err = launch_pdl(k_router_decode<NT>, dim3(rgrid), dim3(RouterCfg<NT>::kWarps * 32), router_smem_bytes(D, n),
                         st, pdl && ws.chain_wait != nullptr, W, D, ws, x, n, ws.route_ready);
    }
    mk.after();
    if (err != cudaSuccess) return err;
    mk.before();
    err = launch_pdl(k_moe_decode<NT, Q4>, dim3(n_sm), dim3(GateUpCfg<NT>::kThreads), s1, st, pdl, W, D, ws, x, n);
    mk.after();
    if (err != cudaSuccess) return err;
    const int64_t nel = (int64_t)n * D.H;
    mk.before();
    if (ws.steer_v)
        err = launch_pdl(k_combine_steer_decode, dim3((unsigned)n), dim3(kSteerThreads), 0, st, pdl, D, ws, out, n);
    else
        err = launch_pdl(k_combine_decode, dim3((unsigned)((nel + 255) / 256)), dim3(256), 0, st, pdl, D, ws, out, n);
    mk.after();
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

int decode_launches() { return 3; }
// CTAs of the decode plan's combine launch for n tokens (what a chained layer counts).
unsigned decode_combine_ctas(const Dims& D, int n, bool steer) {
    return steer ? (unsigned)n : (unsigned)(((int64_t)n * D.H + 255) / 256);
}
const char* decode_kernel_name(int i) { return (i >= 0 && i < 3) ? kDecodeKernels[i] : nullptr; }

// Dynamic shared memory of the larger decode kernel for n tokens, plus its
// static shared memory (pipeline barriers, routing table).
size_t decode_smem_bytes(const Dims& D, int n) {
    size_t a;
    if (n <= 1) a = gateup_smem_bytes<1>(D, n);
    else if (n <= 2) a = gateup_smem_bytes<2>(D, n);
    else if (n <= 4) a = gateup_smem_bytes<4>(D, n);
    else a = gateup_smem_bytes<8>(D, n);
    size_t need = a + sizeof(Pipe) + sizeof(Routing) + 512;   // + the kernel's other static shared memory
    const size_t r = router_smem_bytes(D, n) + sizeof(float) * 8 * 1024 + 64;
    return r > need ? r : need;
}

cudaError_t launch_decode(const Weights& W, const Dims& D, const DecodeWs& ws, const void* x, int n, float* out,
                          int n_sm, cudaStream_t st, cudaEvent_t const* ev, const int32_t* ids_in,
                          const float* wts_in) {
    if (D.q4) {
        if (n <= 1) return launch_decode_t<1, true>(W, D, ws, x, n, out, n_sm, st, ev, ids_in, wts_in);
        if (n <= 2) return launch_decode_t<2, true>(W, D, ws, x, n, out, n_sm, st, ev, ids_in, wts_in);
        if (n <= 4) return launch_decode_t<4, true>(W, D, ws, x, n, out, n_sm, st, ev, ids_in, wts_in);
        return launch_decode_t<8, true>(W, D, ws, x, n, out, n_sm, st, ev, ids_in, wts_in);
    }
    if (n <= 1) return launch_decode_t<1, false>(W, D, ws, x, n, out, n_sm, st, ev, ids_in, wts_in);
    if (n <= 2) return launch_decode_t<2, false>(W, D, ws, x, n, out, n_sm, st, ev, ids_in, wts_in);
    if (n <= 4) return launch_decode_t<4, false>(W, D, ws, x, n, out, n_sm, st, ev, ids_in, wts_in);
    return launch_decode_t<8, false>(W, D, ws, x, n, out, n_sm, st, ev, ids_in, wts_in);
}

// Probe of the down kernel: caller h [n][I] binary32 -> the workspace's h pieces (routed layout at slots
// t * k, or the shared layout) and, for the routed layout, the per-16 sums of the pieces.
__global__ void k_probe_h(const float* h, int n, int I, int k, int shared, uint16_t* hb_rt, float* hsum_rt,
                          uint16_t* hb_sh) {
    const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // one 16-column block
    if (q >= (int64_t)n * (I / 16)) return;
    const int tk = (int)(q / (I / 16)), b = (int)(q % (I / 16));
    float s = 0.f;
    for (int j = 0; j < 16; ++j) {
        const int c = 16 * b + j;
        const float v = h[(int64_t)tk * I + c];
        const uint32_t hi = bf16_bits(v);
        const float hf = __uint_as_float(hi << 16);
        const uint32_t lo = bf16_bits(v - hf);
        if (shared) {
            uint16_t* d = hb_sh + (size_t)tk * 2 * I;
            d[hsh_index(c, 0)] = (uint16_t)hi;
            d[hsh_index(c, 1)] = (uint16_t)lo;
        } else {
            uint16_t* d = hb_rt + (size_t)tk * k * 2 * I;
            d[hrt_index(c, 0)] = (uint16_t)hi;
            d[hrt_index(c, 1)] = (uint16_t)lo;
            s += hf + __uint_as_float(lo << 16);
        }
    }
    if (!shared) hsum_rt[(size_t)tk * k * (I / 16) + b] = s;
}

template <int NT, bool Q4>
cudaError_t launch_probe_decode_t(const Weights& W, const Dims& D, const DecodeWs& ws, int which, const void* in,
                                  int n, int n_sm, cudaStream_t st) {
    cudaError_t err;
    if ((err = configure(k_moe_decode<NT, Q4>)) != cudaSuccess) return err;
    DecodeWs w = ws;
    if (which == 0) {   // gate and up projections of x = in
        w.stages = 1;
        k_moe_decode<NT, Q4><<<n_sm, GateUpCfg<NT>::kThreads, gateup_smem_bytes<NT>(D, n), st>>>(W, D, w, in, n);
        return cudaGetLastError();
    }
    const int64_t nb = (int64_t)n * (D.I / 16);
    k_probe_h<<<(unsigned)((nb + 127) / 128), 128, 0, st>>>(reinterpret_cast<const float*>(in), n, D.I, D.k,
                                                            ws.probe == 2, ws.hb_rt, ws.hsum_rt, ws.hb_sh);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    w.stages = 2;   // down projection of h = in
    k_moe_decode<NT, Q4><<<n_sm, GateUpCfg<NT>::kThreads, gateup_smem_bytes<NT>(D, n), st>>>(W, D, w, nullptr, n);
    return cudaGetLastError();
}

// Inspection: the decode plan's projection kernels with every token routed to
// one expert (ws.probe set by the caller), raw accumulators to ws.probe_out.
cudaError_t launch_probe_decode(const Weights& W, const Dims& D, const DecodeWs& ws, int which, const void* in, int n,
                                int n_sm, cudaStream_t st) {
    if (D.q4) {
        if (n <= 1) return launch_probe_decode_t<1, true>(W, D, ws, which, in, n, n_sm, st);
        if (n <= 2) return launch_probe_decode_t<2, true>(W, D, ws, which, in, n, n_sm, st);
        if (n <= 4) return launch_probe_decode_t<4, true>(W, D, ws, which, in, n, n_sm, st);
        return launch_probe_decode_t<8, true>(W, D, ws, which, in, n, n_sm, st);
    }
    if (n <= 1) return launch_probe_decode_t<1, false>(W, D, ws, which, in, n, n_sm, st);
    if (n <= 2) return launch_probe_decode_t<2, false>(W, D, ws, which, in, n, n_sm, st);
    if (n <= 4) return launch_probe_decode_t<4, false>(W, D, ws, which, in, n, n_sm, st);
    return launch_probe_decode_t<8, false>(W, D, ws, which, in, n, n_sm, st);
}

template <int NT>
cudaError_t launch_route_t(const Weights& W, const Dims& D, const DecodeWs& ws, const void* x, int n,
                           cudaStream_t st) {
    cudaError_t err;
    const size_t s0 = router_smem_bytes(D, n);
    if ((err = configure(k_router_decode<NT>)) != cudaSuccess) return err;
    k_router_decode<NT><<<(D.E + kRE - 1) / kRE, RouterCfg<NT>::kWarps * 32, s0, st>>>(W, D, ws, x, n, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_route(const Weights& W, const Dims& D, const DecodeWs& ws, const void* x, int n,
                         cudaStream_t st) {
    if (n <= 1) return launch_route_t<1>(W, D, ws, x, n, st);
    if (n <= 2) return launch_route_t<2>(W, D, ws, x, n, st);
    if (n <= 4) return launch_route_t<4>(W, D, ws, x, n, st);
    return launch_route_t<8>(W, D, ws, x, n, st);
}

}  // namespace ds4
