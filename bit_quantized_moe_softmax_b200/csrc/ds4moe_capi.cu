// ds4moe_capi.cu -- the C ABI (include/ds4moe.h): handle, buffer layout,
// argument checks, loading, and the launch of the decode and prefill plans.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/ds4moe.h"
#include "ds4moe_internal.cuh"

namespace ds4 {
__global__ void k_pack_q2k(const float* w, int64_t n_blocks, uint8_t* out);
__global__ void k_pack_iq2(const float* w, int64_t n_blocks, const uint8_t* grid, uint8_t* out);
__global__ void k_repack_iq2(const uint8_t* src, int R, int C, uint8_t* qs, uint16_t* dd);
__global__ void k_repack_q2(const uint8_t* src, int R, int C, uint8_t* q, uint32_t* sc, uint32_t* dd);
__global__ void k_repack_bf16(const uint4* src, int R, int C, uint4* dst);
__global__ void k_pack_q4k(const float* w, int64_t n_blocks, uint8_t* out);
__global__ void k_repack_q4(const uint8_t* src, int R, int C, int mode, uint8_t* q, uint32_t* sc, uint32_t* dd);
__global__ void k_dequant_q4(const uint8_t* q, const uint32_t* sc, const uint32_t* dd, int R, int C, int mode,
                             float* out_f, __nv_bfloat16* out_b);
__global__ void k_interleave_router(const float* W, int E, int H, float* W2);
__global__ void k_dequant_iq2(const uint8_t* qs, const uint16_t* dd, const uint8_t* grid, int R, int C, float* out_f,
                              __nv_bfloat16* out_b);
__global__ void k_dequant_q2(const uint8_t* q, const uint32_t* sc, const uint32_t* dd, int R, int C, float* out_f,
                             __nv_bfloat16* out_b);
__global__ void k_dequant_bf16_tiles(const __nv_bfloat16* t, int R, int C, float* out_f, __nv_bfloat16* out_b);
cudaError_t launch_decode(const Weights& W, const Dims& D, const DecodeWs& ws, const void* x, int n, float* out,
                          int n_sm, cudaStream_t st, cudaEvent_t const* ev, const int32_t* ids_in = nullptr,
                          const float* wts_in = nullptr);
cudaError_t launch_combine_slots(const float* y, const float* w, const float* base, int n, int k, int H, float* out,
                                 cudaStream_t st);
int decode_launches();
const char* decode_kernel_name(int i);
size_t decode_smem_bytes(const Dims& D, int n);
cudaError_t launch_route(const Weights& W, const Dims& D, const DecodeWs& ws, const void* x, int n,
                         cudaStream_t st);
cudaError_t launch_prefill(const Weights& W, const Dims& D, const PrefillWs& ws, const void* x, int n, float* out,
                           int n_sm, cudaStream_t st, cudaEvent_t const* ev, const int32_t* ids_in = nullptr,
                           const float* wts_in = nullptr);
cudaError_t launch_route_prefill(const Weights& W, const Dims& D, const PrefillWs& ws, const void* x, int n,
                                 cudaStream_t st);
cudaError_t launch_wait_selftest(uint32_t* err, cudaStream_t st);
unsigned decode_combine_ctas(const Dims& D, int n, bool steer);
cudaError_t launch_grid_tables(const uint8_t* grid, uint32_t* gtab, uint32_t* rows, cudaStream_t st);
cudaError_t launch_permutation(const Dims& D, const PrefillWs& ws, const int32_t* ids, int n, cudaStream_t st);
cudaError_t launch_probe_decode(const Weights& W, const Dims& D, const DecodeWs& ws, int which, const void* in, int n,
                                int n_sm, cudaStream_t st);
cudaError_t launch_probe_gemm(const Weights& W, const Dims& D, const PrefillWs& ws, int which, int e,
                              const void* in, int n, float* out, int n_sm, cudaStream_t st);
int prefill_launches(const Dims& D);
const char* prefill_kernel_name(const Dims& D, int i);
size_t gemm_smem_bytes();
size_t gemm_static_smem_bytes();
}  // namespace ds4

using namespace ds4;

// Scratch of ds4moe_route_noalloc: a 64-word header (word 0: the device error
// word, kept until ds4moe_get_device_error reads it; words 1.. : the router's
// ticket and task counters, cleared before every call) followed by the logits
// of up to kNoAllocLogits (token, expert) pairs.  kNoAllocLogits = 8192 is the
// largest n_tokens * n_experts a handle can ask for (decode_max <= 8 tokens,
// n_experts <= 1024), so the size check in the entry point is a defensive one.
// One copy per device, for the life of the process; its device address is
// looked up once per device (noalloc_scratch) and kept in g_noalloc_addr.
constexpr int kNoAllocHeader = 64;
constexpr int kNoAllocLogits = 8192;
constexpr int kNoAllocDevices = 64;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocHeader + kNoAllocLogits];
static std::mutex g_noalloc_mu;
static float* g_noalloc_addr[kNoAllocDevices] = {};

namespace {

thread_local std::string g_err;

ds4moe_status fail(ds4moe_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
ds4moe_status fail(ds4moe_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

ds4moe_status cuda_fail(cudaError_t e, const char* what) {
    return fail(DS4MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }
bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

struct WsLayout {
    size_t hdr, logits, ids, wts, hb_rt, hsum_rt, hb_sh, y_rt, y_sh, x_stage, out_stage;
    size_t x_slot, out_slot;   // bytes of one of the two staging slots of the host-buffer calls
    // prefill plan (capacity > decode_max only)
    size_t p_logits, p_ids, p_wts, p_blk_cnt, p_blk_off, p_counts, p_offs, p_mtp, p_pos, p_slot, p_xb, p_Xp, p_Hb,
        p_Hs, p_Y, p_Ys;
    size_t total;
};

}  // namespace

struct ds4moe {
    ds4moe_shape shape;
    Dims D;
    int decode_max;
    int n_sm;
    // weight buffer layout
    size_t off_grid, off_gtab, off_gtab_rows, off_Wr, off_Wr2, off_br, off_steer, off_gate_qs, off_gate_d, off_up_qs, off_up_d, off_down_q, off_down_sc,
        off_down_dd, off_sh_gate, off_sh_up, off_sh_down, weight_bytes;
    size_t iq2_qs_stride, iq2_d_stride, q2_q_stride, q2_sc_stride, q2_dd_stride;
    // 4-bit layers: codes at off_gate_qs / off_up_qs / off_down_q, scale and (d, dmin) words here
    size_t off_gate_sc4 = 0, off_up_sc4 = 0, off_down_sc4 = 0, off_gate_dd4 = 0, off_up_dd4 = 0, off_down_dd4 = 0;
    size_t q4_q_stride = 0, q4_sc_stride = 0, q4_dd_stride = 0;
    uint8_t* weights = nullptr;
    uint8_t* ws = nullptr;
    size_t ws_bytes = 0;
    WsLayout L{};
    std::vector<uint8_t> loaded;
    bool grid_set = false, router_set = false, shared_set = false;
    bool steer_on = false;   // directional steering of the layer output (ds4moe_set_steering)
    float steer_F = 0.f;
    // host-buffer calls: upload / download streams (created on first use) and,
    // per staging slot, the events of its upload, its forward and its download
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t ev_in[2] = {}, ev_done[2] = {}, ev_out[2] = {};
    int slot = 0;

    ~ds4moe() { release_host_streams(); }
    void release_host_streams() {
        if (up) cudaStreamSynchronize(up);
        if (down) cudaStreamSynchronize(down);
        for (int i = 0; i < 2; ++i) {
            if (ev_in[i]) cudaEventDestroy(ev_in[i]);
            if (ev_done[i]) cudaEventDestroy(ev_done[i]);
            if (ev_out[i]) cudaEventDestroy(ev_out[i]);
            ev_in[i] = ev_done[i] = ev_out[i] = nullptr;
        }
        if (up) cudaStreamDestroy(up);
        if (down) cudaStreamDestroy(down);
        up = down = nullptr;
    }
    cudaError_t host_streams() {
        if (up) return cudaSuccess;
        cudaError_t e = cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking);
        for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&ev_in[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_done[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_out[i], cudaEventDisableTiming);
        }
        if (e != cudaSuccess) release_host_streams();
        return e;
    }

    WsLayout layout(int cap) const {
        WsLayout w{};
        const size_t H = D.H, I = D.I, E = D.E, k = D.k;
        const size_t nd = (size_t)(cap < decode_max ? cap : decode_max);
        size_t o = 0;
        w.hdr = o; o += 1024;   // 256 words: control words 0..7, gate/up completion counters from word 16
        w.logits = o; o += align256(nd * E * 4);
        w.ids = o; o += align256(nd * k * 4);
        w.wts = o; o += align256(nd * k * 4);
        w.hb_rt = o; o += align256(nd * k * I * 2 * 2);   // two bf16 pieces
        w.hsum_rt = o; o += align256(nd * k * (I / 16) * 4);
        w.hb_sh = o; o += align256(nd * I * 2 * 2);
        w.y_rt = o; o += align256(nd * k * H * 4);
        w.y_sh = o; o += align256(nd * H * 4);
        w.x_slot = align256((size_t)cap * H * (D.act_bf16 ? 2 : 4));
        w.out_slot = align256((size_t)cap * H * 4);
        w.x_stage = o; o += 2 * w.x_slot;
        w.out_stage = o; o += 2 * w.out_slot;
        if (cap > decode_max) {
            const size_t N = cap, NK = N * k, nblk = (NK + 1023) / 1024;
            w.p_logits = o; o += align256(N * E * 4);
            w.p_ids = o; o += align256(NK * 4);
            w.p_wts = o; o += align256(NK * 4);
            w.p_blk_cnt = o; o += align256(nblk * E * 4);
            w.p_blk_off = o; o += align256(nblk * E * 4);
            w.p_counts = o; o += align256(E * 4);
            w.p_offs = o; o += align256((E + 1) * 4);
            w.p_mtp = o; o += align256((E + 1) * 4);
            w.p_pos = o; o += align256(NK * 4);
            w.p_slot = o; o += align256(NK * 4);
            w.p_xb = o; o += align256(N * H * 2);
            w.p_Xp = o; o += align256(NK * H * 2);
            w.p_Hb = o; o += align256(NK * I * 2);
            w.p_Hs = o; o += align256(N * I * 2);
            w.p_Y = o; o += align256(NK * H * 4);
            w.p_Ys = o; o += align256(N * H * 4);
        }
        w.total = o;
        return w;
    }

    Weights weights_view() const {
        Weights W{};
        const uint8_t* b = weights;
        W.grid_u8 = b + off_grid;
        W.gtab = reinterpret_cast<const uint32_t*>(b + off_gtab);
        W.gtab_rows = reinterpret_cast<const uint32_t*>(b + off_gtab_rows);
        W.W_r = reinterpret_cast<const float*>(b + off_Wr);
        W.W_r2 = shape.max_tokens > decode_max ? reinterpret_cast<const float*>(b + off_Wr2) : nullptr;
        W.b_r = shape.has_bias ? reinterpret_cast<const float*>(b + off_br) : nullptr;
        W.gate_qs = b + off_gate_qs;
        W.gate_d = reinterpret_cast<const uint16_t*>(b + off_gate_d);
        W.up_qs = b + off_up_qs;
        W.up_d = reinterpret_cast<const uint16_t*>(b + off_up_d);
        W.down_q = b + off_down_q;
        W.down_sc = reinterpret_cast<const uint32_t*>(b + off_down_sc);
        W.down_dd = reinterpret_cast<const uint32_t*>(b + off_down_dd);
        W.sh_gate = reinterpret_cast<const __nv_bfloat16*>(b + off_sh_gate);
        W.sh_up = reinterpret_cast<const __nv_bfloat16*>(b + off_sh_up);
        W.sh_down = reinterpret_cast<const __nv_bfloat16*>(b + off_sh_down);
        W.iq2_qs_stride = iq2_qs_stride;
        W.iq2_d_stride = iq2_d_stride;
        W.q2_q_stride = q2_q_stride;
        W.q2_sc_stride = q2_sc_stride;
        W.q2_dd_stride = q2_dd_stride;
        if (D.q4) {
            W.gate_sc4 = reinterpret_cast<const uint32_t*>(b + off_gate_sc4);
            W.up_sc4 = reinterpret_cast<const uint32_t*>(b + off_up_sc4);
            W.down_sc4 = reinterpret_cast<const uint32_t*>(b + off_down_sc4);
            W.gate_dd4 = reinterpret_cast<const uint32_t*>(b + off_gate_dd4);
            W.up_dd4 = reinterpret_cast<const uint32_t*>(b + off_up_dd4);
            W.down_dd4 = reinterpret_cast<const uint32_t*>(b + off_down_dd4);
            W.q4_q_stride = q4_q_stride;
            W.q4_sc_stride = q4_sc_stride;
            W.q4_dd_stride = q4_dd_stride;
        }
        return W;
    }

    DecodeWs decode_ws() const {
        DecodeWs w{};
        uint32_t* hdr = reinterpret_cast<uint32_t*>(ws + L.hdr);
        w.err = hdr + 0;
        w.ticket = hdr + 1;
        w.queue = hdr + 2;
        w.queue_rt = hdr + 3;
        w.done = hdr + 4;
        w.grid_refused = hdr + 6;
        w.route_ready = hdr + 7;
        w.gu_done = hdr + 16;   // word 10: this layer's count of combine CTAs in a chained forward
        w.stages = 3;
        w.logits = reinterpret_cast<float*>(ws + L.logits);
        w.ids = reinterpret_cast<int32_t*>(ws + L.ids);
        w.wts = reinterpret_cast<float*>(ws + L.wts);
        w.hb_rt = reinterpret_cast<uint16_t*>(ws + L.hb_rt);
        w.hsum_rt = reinterpret_cast<float*>(ws + L.hsum_rt);
        w.hb_sh = reinterpret_cast<uint16_t*>(ws + L.hb_sh);
        w.y_rt = reinterpret_cast<float*>(ws + L.y_rt);
        w.y_sh = reinterpret_cast<float*>(ws + L.y_sh);
        return w;
    }

    PrefillWs prefill_ws() const {
        PrefillWs w{};
        w.logits = reinterpret_cast<float*>(ws + L.p_logits);
        w.ids = reinterpret_cast<int32_t*>(ws + L.p_ids);
        w.wts = reinterpret_cast<float*>(ws + L.p_wts);
        w.blk_cnt = reinterpret_cast<int32_t*>(ws + L.p_blk_cnt);
        w.blk_off = reinterpret_cast<int32_t*>(ws + L.p_blk_off);
        w.counts = reinterpret_cast<int32_t*>(ws + L.p_counts);
        w.offs = reinterpret_cast<int32_t*>(ws + L.p_offs);
        w.mt_prefix = reinterpret_cast<int32_t*>(ws + L.p_mtp);
        w.pos_of_slot = reinterpret_cast<int32_t*>(ws + L.p_pos);
        w.slot_of_pos = reinterpret_cast<int32_t*>(ws + L.p_slot);
        w.xb = reinterpret_cast<__nv_bfloat16*>(ws + L.p_xb);
        w.Xp = reinterpret_cast<__nv_bfloat16*>(ws + L.p_Xp);
        w.Hb = reinterpret_cast<__nv_bfloat16*>(ws + L.p_Hb);
        w.Hs = reinterpret_cast<__nv_bfloat16*>(ws + L.p_Hs);
        w.Y = reinterpret_cast<float*>(ws + L.p_Y);
        w.Ys = reinterpret_cast<float*>(ws + L.p_Ys);
        w.err = reinterpret_cast<uint32_t*>(ws + L.hdr);
        w.grid_refused = reinterpret_cast<uint32_t*>(ws + L.hdr) + 6;
        return w;
    }

    bool ready(std::string* why) const {
        if (!weights) { *why = "buffers not bound"; return false; }
        if (!ws) { *why = "workspace not bound"; return false; }
        if (!grid_set && !D.q4) { *why = "grid not set"; return false; }
        if (!router_set) { *why = "router not set"; return false; }
        if (shape.has_shared && !shared_set) { *why = "shared expert not set"; return false; }
        for (size_t e = 0; e < loaded.size(); ++e)
            if (!loaded[e]) { *why = "expert " + std::to_string(e) + " not loaded"; return false; }
        return true;
    }
};

extern "C" {

const char* ds4moe_last_error(void) { return g_err.c_str(); }

ds4moe_status ds4moe_create(const ds4moe_shape* s, ds4moe_t** out) {
    if (!s || !out) return fail(DS4MOE_ERR_ARG, "create: NULL argument");
    *out = nullptr;
    if (s->hidden < 256 || s->hidden % 256) return fail(DS4MOE_ERR_SHAPE, "hidden %d: need a multiple of 256", s->hidden);
    if (!(s->inter == 128 || (s->inter >= 256 && s->inter % 256 == 0)))
        return fail(DS4MOE_ERR_SHAPE, "inter %d: need 128 or a multiple of 256", s->inter);
    if (s->n_experts < 1 || s->n_experts > 1024) return fail(DS4MOE_ERR_SHAPE, "n_experts %d: need 1..1024", s->n_experts);
    if (s->top_k < 1 || s->top_k > 16 || s->top_k > s->n_experts)
        return fail(DS4MOE_ERR_SHAPE, "top_k %d: need 1..min(16, n_experts)", s->top_k);
    if (s->max_tokens < 1) return fail(DS4MOE_ERR_SHAPE, "max_tokens %d: need >= 1", s->max_tokens);
    if (s->act_dtype != DS4MOE_ACT_F32 && s->act_dtype != DS4MOE_ACT_BF16)
        return fail(DS4MOE_ERR_SHAPE, "act_dtype %d unknown", s->act_dtype);
    if (s->decode_max < 0 || s->decode_max > 8) return fail(DS4MOE_ERR_SHAPE, "decode_max %d: need 0..8", s->decode_max);
    if (s->expert_bits != 0 && s->expert_bits != 2 && s->expert_bits != 4)
        return fail(DS4MOE_ERR_SHAPE, "expert_bits %d: need 0, 2 or 4", s->expert_bits);
    if (s->expert_bits == 4 && s->inter % 256)
        return fail(DS4MOE_ERR_SHAPE, "expert_bits 4: inter %d not a multiple of 256", s->inter);
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
    int n_sm = 0;
    ce = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (ce != cudaSuccess) return cuda_fail(ce, "cudaDeviceGetAttribute");

    ds4moe* h = new ds4moe();
    h->shape = *s;
    h->D.H = s->hidden;
    h->D.I = s->inter;
    h->D.E = s->n_experts;
    h->D.k = s->top_k;
    h->D.has_shared = s->has_shared ? 1 : 0;
    h->D.act_bf16 = s->act_dtype == DS4MOE_ACT_BF16;
    h->D.q4 = s->expert_bits == 4;
    h->decode_max = s->decode_max ? s->decode_max : 8;
    h->n_sm = n_sm;
    {
        int smem_optin = 0;
        ce = cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (ce != cudaSuccess) { delete h; return cuda_fail(ce, "cudaDeviceGetAttribute"); }
        size_t need = decode_smem_bytes(h->D, h->decode_max);
        const size_t gemm_need = gemm_smem_bytes() + gemm_static_smem_bytes();
        if (s->max_tokens > h->decode_max && gemm_need > need) need = gemm_need;
        if (need > (size_t)smem_optin) {
            delete h;
            return fail(DS4MOE_ERR_SHAPE, "the plan needs %zu bytes of shared memory per CTA (device: %d); "
                        "lower decode_max or hidden", need, smem_optin);
        }
    }
    const size_t H = s->hidden, I = s->inter, E = s->n_experts;
    const size_t nsb_down = I >= 256 ? I / 256 : 1;
    h->iq2_qs_stride = I * H / 4;
    h->iq2_d_stride = I * H / 256;
    h->q2_q_stride = H * I / 4;
    h->q2_sc_stride = H * I / 64;
    h->q2_dd_stride = H * nsb_down;
    size_t o = 0;
    h->off_grid = o; o += align256(256 * 8);
    h->off_gtab = o; o += align256((256 + 128 + 4) * 4);
    h->off_gtab_rows = o; o += align256(256 * 64 * 4);
    h->off_Wr = o; o += align256(E * H * 4);
    h->off_Wr2 = o; o += align256(s->max_tokens > h->decode_max ? (E + 1) / 2 * 2 * H * 4 : 0);
    h->off_br = o; o += align256(E * 4);
    h->off_steer = o; o += align256(H * 4);
    if (h->D.q4) {
        // codes 32 bytes, one scale word per (row, 64 columns), one (d, dmin) word per (row, 256 columns)
        h->q4_q_stride = I * H / 2;
        h->q4_sc_stride = I * H / 64;
        h->q4_dd_stride = I * H / 256;
        h->off_gate_qs = o; o += align256(E * h->q4_q_stride);
        h->off_up_qs = o; o += align256(E * h->q4_q_stride);
        h->off_down_q = o; o += align256(E * h->q4_q_stride);
        h->off_gate_sc4 = o; o += align256(E * h->q4_sc_stride * 4);
        h->off_up_sc4 = o; o += align256(E * h->q4_sc_stride * 4);
        h->off_down_sc4 = o; o += align256(E * h->q4_sc_stride * 4);
        h->off_gate_dd4 = o; o += align256(E * h->q4_dd_stride * 4);
        h->off_up_dd4 = o; o += align256(E * h->q4_dd_stride * 4);
        h->off_down_dd4 = o; o += align256(E * h->q4_dd_stride * 4);
        h->off_gate_d = h->off_up_d = h->off_down_sc = h->off_down_dd = 0;
    } else {
        h->off_gate_qs = o; o += align256(E * h->iq2_qs_stride);
        h->off_gate_d = o; o += align256(E * h->iq2_d_stride * 2);
        h->off_up_qs = o; o += align256(E * h->iq2_qs_stride);
        h->off_up_d = o; o += align256(E * h->iq2_d_stride * 2);
        h->off_down_q = o; o += align256(E * h->q2_q_stride);
        h->off_down_sc = o; o += align256(E * h->q2_sc_stride * 4);
        h->off_down_dd = o; o += align256(E * h->q2_dd_stride * 4);
    }
    h->off_sh_gate = o; o += align256(s->has_shared ? I * H * 2 : 0);
    h->off_sh_up = o; o += align256(s->has_shared ? I * H * 2 : 0);
    h->off_sh_down = o; o += align256(s->has_shared ? H * I * 2 : 0);
    h->weight_bytes = o;
    h->loaded.assign(E, 0);
    *out = h;
    g_err.clear();
    return DS4MOE_OK;
}

ds4moe_status ds4moe_destroy(ds4moe_t* h) {
    if (!h) return fail(DS4MOE_ERR_ARG, "destroy: NULL handle");
    delete h;
    return DS4MOE_OK;
}

size_t ds4moe_weight_bytes(const ds4moe_t* h) { return h ? h->weight_bytes : 0; }

size_t ds4moe_workspace_bytes(const ds4moe_t* h, int32_t n_tokens) {
    if (!h || n_tokens < 1) return 0;
    return h->layout(n_tokens).total;
}

ds4moe_status ds4moe_bind(ds4moe_t* h, void* d_weights, size_t weight_bytes, void* d_workspace, size_t ws_bytes,
                          void* stream) {
    if (!h || !d_weights) return fail(DS4MOE_ERR_ARG, "bind: NULL argument");
    if (!d_workspace && ws_bytes != 0) return fail(DS4MOE_ERR_ARG, "bind: NULL workspace with a nonzero size");
    if (((uintptr_t)d_weights & 255) || ((uintptr_t)d_workspace & 255))
        return fail(DS4MOE_ERR_ALIGN, "bind: buffers must be 256-byte aligned");
    if (weight_bytes < h->weight_bytes)
        return fail(DS4MOE_ERR_ARG, "bind: weight buffer %zu bytes < %zu", weight_bytes, h->weight_bytes);
    WsLayout L = h->layout(h->shape.max_tokens);
    if (d_workspace && ws_bytes < L.total)
        return fail(DS4MOE_ERR_ARG, "bind: workspace %zu bytes < %zu", ws_bytes, L.total);
    // pipelined host-buffer calls still in flight use the old staging slots
    ds4moe_status hs = ds4moe_host_sync(h);
    if (hs != DS4MOE_OK) return hs;
    h->slot = 0;
    if (d_workspace) {
        cudaError_t ce = cudaMemsetAsync(static_cast<uint8_t*>(d_workspace) + L.hdr, 0, L.logits - L.hdr,
                                         (cudaStream_t)stream);
        if (ce != cudaSuccess) return cuda_fail(ce, "bind: cudaMemsetAsync");
    }
    h->weights = static_cast<uint8_t*>(d_weights);
    h->ws = static_cast<uint8_t*>(d_workspace);
    h->ws_bytes = ws_bytes;
    h->L = L;
    std::fill(h->loaded.begin(), h->loaded.end(), 0);
    h->grid_set = h->router_set = h->shared_set = false;
    return DS4MOE_OK;
}

ds4moe_status ds4moe_pack_q2k(const float* d_w, int64_t n, void* d_blocks, void* stream) {
    if (!d_w || !d_blocks) return fail(DS4MOE_ERR_ARG, "pack_q2k: NULL argument");
    if (n <= 0 || n % kQK) return fail(DS4MOE_ERR_ARG, "pack_q2k: n_weights %lld not a positive multiple of 256", (long long)n);
    if (!aligned16(d_w)) return fail(DS4MOE_ERR_ALIGN, "pack_q2k: weights not 16-byte aligned");
    const int64_t nb = n / kQK;
    k_pack_q2k<<<(unsigned)((nb + 127) / 128), 128, 0, (cudaStream_t)stream>>>(d_w, nb, (uint8_t*)d_blocks);
    cudaError_t ce = cudaGetLastError();
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "pack_q2k launch");
}

ds4moe_status ds4moe_pack_q4k(const float* d_w, int64_t n, void* d_blocks, void* stream) {
    if (!d_w || !d_blocks) return fail(DS4MOE_ERR_ARG, "pack_q4k: NULL argument");
    if (n <= 0 || n % kQK) return fail(DS4MOE_ERR_ARG, "pack_q4k: n_weights %lld not a positive multiple of 256", (long long)n);
    if (!aligned16(d_w)) return fail(DS4MOE_ERR_ALIGN, "pack_q4k: weights not 16-byte aligned");
    const int64_t nb = n / kQK;
    k_pack_q4k<<<(unsigned)((nb + 127) / 128), 128, 0, (cudaStream_t)stream>>>(d_w, nb, (uint8_t*)d_blocks);
    cudaError_t ce = cudaGetLastError();
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "pack_q4k launch");
}

ds4moe_status ds4moe_pack_iq2xxs(const float* d_w, int64_t n, const uint8_t* d_grid, void* d_blocks, void* stream) {
    if (!d_w || !d_blocks || !d_grid) return fail(DS4MOE_ERR_ARG, "pack_iq2xxs: NULL argument");
    if (n <= 0 || n % kQK) return fail(DS4MOE_ERR_ARG, "pack_iq2xxs: n_weights %lld not a positive multiple of 256", (long long)n);
    if (!aligned16(d_w)) return fail(DS4MOE_ERR_ALIGN, "pack_iq2xxs: weights not 16-byte aligned");
    const int64_t nb = n / kQK;
    k_pack_iq2<<<(unsigned)((nb + 3) / 4), 128, 0, (cudaStream_t)stream>>>(d_w, nb, d_grid, (uint8_t*)d_blocks);
    cudaError_t ce = cudaGetLastError();
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "pack_iq2xxs launch");
}

ds4moe_status ds4moe_set_grid(ds4moe_t* h, const uint8_t* d_grid, void* stream) {
    if (!h || !d_grid) return fail(DS4MOE_ERR_ARG, "set_grid: NULL argument");
    if (!h->weights) return fail(DS4MOE_ERR_NOT_READY, "set_grid: buffers not bound");
    cudaError_t ce = cudaMemcpyAsync(h->weights + h->off_grid, d_grid, 256 * 8, cudaMemcpyDeviceToDevice,
                                     (cudaStream_t)stream);
    if (ce == cudaSuccess)
        ce = launch_grid_tables(h->weights + h->off_grid, reinterpret_cast<uint32_t*>(h->weights + h->off_gtab),
                                reinterpret_cast<uint32_t*>(h->weights + h->off_gtab_rows),
                                (cudaStream_t)stream);
    if (ce != cudaSuccess) return cuda_fail(ce, "set_grid copy");
    h->grid_set = true;
    return DS4MOE_OK;
}

ds4moe_status ds4moe_set_router(ds4moe_t* h, const float* d_W, const float* d_bias, void* stream) {
    if (!h || !d_W) return fail(DS4MOE_ERR_ARG, "set_router: NULL argument");
    if (!h->weights) return fail(DS4MOE_ERR_NOT_READY, "set_router: buffers not bound");
    if (h->shape.has_bias && !d_bias) return fail(DS4MOE_ERR_ARG, "set_router: has_bias set but bias is NULL");
    if (!h->shape.has_bias && d_bias) return fail(DS4MOE_ERR_ARG, "set_router: bias given but has_bias is 0");
    cudaStream_t st = (cudaStream_t)stream;
    const size_t E = h->D.E, H = h->D.H;
    cudaError_t ce = cudaMemcpyAsync(h->weights + h->off_Wr, d_W, E * H * 4, cudaMemcpyDeviceToDevice, st);
    if (ce == cudaSuccess && h->shape.max_tokens > h->decode_max) {
        const int64_t m = (int64_t)(E + 1) / 2 * H;
        k_interleave_router<<<(unsigned)((m + 255) / 256), 256, 0, st>>>(
            reinterpret_cast<const float*>(h->weights + h->off_Wr), (int)E, (int)H,
            reinterpret_cast<float*>(h->weights + h->off_Wr2));
        ce = cudaGetLastError();
    }
    if (ce == cudaSuccess && d_bias)
        ce = cudaMemcpyAsync(h->weights + h->off_br, d_bias, E * 4, cudaMemcpyDeviceToDevice, st);
    if (ce != cudaSuccess) return cuda_fail(ce, "set_router copy");
    h->router_set = true;
    return DS4MOE_OK;
}

ds4moe_status ds4moe_set_steering(ds4moe_t* h, const float* d_v, float F, void* stream) {
    if (!h) return fail(DS4MOE_ERR_ARG, "set_steering: NULL handle");
    if (!h->weights) return fail(DS4MOE_ERR_NOT_READY, "set_steering: buffers not bound");
    if (!d_v || F == 0.f) {   // off
        h->steer_on = false;
        h->steer_F = 0.f;
        return DS4MOE_OK;
    }
    if (h->D.H > 4096) return fail(DS4MOE_ERR_SHAPE, "set_steering: hidden %d above 4096", h->D.H);
    if (!(F == F) || F - F != 0.f) return fail(DS4MOE_ERR_ARG, "set_steering: F not finite");
    cudaError_t ce = cudaMemcpyAsync(h->weights + h->off_steer, d_v, (size_t)h->D.H * 4, cudaMemcpyDeviceToDevice,
                                     (cudaStream_t)stream);
    if (ce != cudaSuccess) return cuda_fail(ce, "set_steering copy");
    h->steer_on = true;
    h->steer_F = F;
    return DS4MOE_OK;
}

ds4moe_status ds4moe_set_expert(ds4moe_t* h, int32_t e, const void* d_gate, const void* d_up, const void* d_down,
                                void* stream) {
    if (!h || !d_gate || !d_up || !d_down) return fail(DS4MOE_ERR_ARG, "set_expert: NULL argument");
    if (!h->weights) return fail(DS4MOE_ERR_NOT_READY, "set_expert: buffers not bound");
    if (e < 0 || e >= h->D.E) return fail(DS4MOE_ERR_ARG, "set_expert: expert %d out of range", e);
    cudaStream_t st = (cudaStream_t)stream;
    const int H = h->D.H, I = h->D.I;
    if (h->D.q4) {
        const int64_t nsteps = (int64_t)I * H / 64;   // (row, 64-column step) pieces of each matrix
        const unsigned g = (unsigned)((nsteps + 255) / 256);
        uint8_t* b = h->weights;
        const size_t qo = e * h->q4_q_stride, so = e * h->q4_sc_stride, dof = e * h->q4_dd_stride;
        k_repack_q4<<<g, 256, 0, st>>>((const uint8_t*)d_gate, I, H, 0, b + h->off_gate_qs + qo,
                                       reinterpret_cast<uint32_t*>(b + h->off_gate_sc4) + so,
                                       reinterpret_cast<uint32_t*>(b + h->off_gate_dd4) + dof);
        k_repack_q4<<<g, 256, 0, st>>>((const uint8_t*)d_up, I, H, 0, b + h->off_up_qs + qo,
                                       reinterpret_cast<uint32_t*>(b + h->off_up_sc4) + so,
                                       reinterpret_cast<uint32_t*>(b + h->off_up_dd4) + dof);
        k_repack_q4<<<g, 256, 0, st>>>((const uint8_t*)d_down, H, I, 1, b + h->off_down_q + qo,
                                       reinterpret_cast<uint32_t*>(b + h->off_down_sc4) + so,
                                       reinterpret_cast<uint32_t*>(b + h->off_down_dd4) + dof);
        cudaError_t ce = cudaGetLastError();
        if (ce != cudaSuccess) return cuda_fail(ce, "set_expert launch");
        h->loaded[e] = 1;
        return DS4MOE_OK;
    }
    const int64_t nb = (int64_t)I * H / kQK;
    const unsigned g1 = (unsigned)((nb * 8 + 255) / 256);
    k_repack_iq2<<<g1, 256, 0, st>>>((const uint8_t*)d_gate, I, H, h->weights + h->off_gate_qs + e * h->iq2_qs_stride,
                                     reinterpret_cast<uint16_t*>(h->weights + h->off_gate_d) + e * h->iq2_d_stride);
    k_repack_iq2<<<g1, 256, 0, st>>>((const uint8_t*)d_up, I, H, h->weights + h->off_up_qs + e * h->iq2_qs_stride,
                                     reinterpret_cast<uint16_t*>(h->weights + h->off_up_d) + e * h->iq2_d_stride);
    const int64_t npieces = (int64_t)H * (I / 64);
    k_repack_q2<<<(unsigned)((npieces + 255) / 256), 256, 0, st>>>(
        (const uint8_t*)d_down, H, I, h->weights + h->off_down_q + e * h->q2_q_stride,
        reinterpret_cast<uint32_t*>(h->weights + h->off_down_sc) + e * h->q2_sc_stride,
        reinterpret_cast<uint32_t*>(h->weights + h->off_down_dd) + e * h->q2_dd_stride);
    cudaError_t ce = cudaGetLastError();
    if (ce != cudaSuccess) return cuda_fail(ce, "set_expert launch");
    h->loaded[e] = 1;
    return DS4MOE_OK;
}

ds4moe_status ds4moe_set_shared(ds4moe_t* h, const void* d_gate, const void* d_up, const void* d_down, void* stream) {
    if (!h || !d_gate || !d_up || !d_down) return fail(DS4MOE_ERR_ARG, "set_shared: NULL argument");
    if (!h->weights) return fail(DS4MOE_ERR_NOT_READY, "set_shared: buffers not bound");
    if (!h->shape.has_shared) return fail(DS4MOE_ERR_ARG, "set_shared: layer created without a shared expert");
    if (!aligned16(d_gate) || !aligned16(d_up) || !aligned16(d_down))
        return fail(DS4MOE_ERR_ALIGN, "set_shared: matrices must be 16-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    const int H = h->D.H, I = h->D.I;
    const int64_t n8 = (int64_t)I * H / 8;
    const unsigned g = (unsigned)((n8 + 255) / 256);
    k_repack_bf16<<<g, 256, 0, st>>>((const uint4*)d_gate, I, H, (uint4*)(h->weights + h->off_sh_gate));
    k_repack_bf16<<<g, 256, 0, st>>>((const uint4*)d_up, I, H, (uint4*)(h->weights + h->off_sh_up));
    k_repack_bf16<<<g, 256, 0, st>>>((const uint4*)d_down, H, I, (uint4*)(h->weights + h->off_sh_down));
    cudaError_t ce = cudaGetLastError();
    if (ce != cudaSuccess) return cuda_fail(ce, "set_shared launch");
    h->shared_set = true;
    return DS4MOE_OK;
}

static ds4moe_status check_forward(ds4moe_t* h, const void* x, int32_t n, const void* out, const char* who) {
    if (!h) return fail(DS4MOE_ERR_ARG, "%s: NULL handle", who);
    if (n < 0 || n > h->shape.max_tokens)
        return fail(DS4MOE_ERR_ARG, "%s: n_tokens %d outside 0..%d", who, n, h->shape.max_tokens);
    if (n > 0 && (!x || !out)) return fail(DS4MOE_ERR_ARG, "%s: NULL buffer", who);
    std::string why;
    if (!h->ready(&why)) return fail(DS4MOE_ERR_NOT_READY, "%s: %s", who, why.c_str());
    return DS4MOE_OK;
}

static ds4moe_status forward_impl(ds4moe_t* h, const void* d_x, int32_t n, float* d_out, void* const* events,
                                  void* stream, const char* who, bool residual = false,
                                  const int32_t* ids_in = nullptr, const float* wts_in = nullptr) {
    ds4moe_status s = check_forward(h, d_x, n, d_out, who);
    if (s != DS4MOE_OK) return s;
    if (n == 0) return DS4MOE_OK;
    if (!aligned16(d_x) || !aligned16(d_out)) return fail(DS4MOE_ERR_ALIGN, "%s: x and out must be 16-byte aligned", who);
    if (residual) {   // out is written while x is still read: the ranges may not overlap
        const uintptr_t xa = reinterpret_cast<uintptr_t>(d_x), oa = reinterpret_cast<uintptr_t>(d_out);
        const size_t xbytes = (size_t)n * h->D.H * (h->D.act_bf16 ? 2 : 4), obytes = (size_t)n * h->D.H * 4;
        if (xa < oa + obytes && oa < xa + xbytes) return fail(DS4MOE_ERR_ARG, "%s: x and out overlap", who);
    }
    cudaStream_t st = (cudaStream_t)stream;
    cudaEvent_t const* ev = reinterpret_cast<cudaEvent_t const*>(events);
    cudaError_t ce;
    if (n <= h->decode_max) {
        DecodeWs ws = h->decode_ws();
        ws.xres = residual ? d_x : nullptr;
        ws.steer_v = h->steer_on ? reinterpret_cast<const float*>(h->weights + h->off_steer) : nullptr;
        ws.steer_F = h->steer_F;
        ce = launch_decode(h->weights_view(), h->D, ws, d_x, n, d_out, h->n_sm, st, ev, ids_in, wts_in);
    } else {
        PrefillWs ws = h->prefill_ws();
        ws.xres = residual ? d_x : nullptr;
        ws.steer_v = h->steer_on ? reinterpret_cast<const float*>(h->weights + h->off_steer) : nullptr;
        ws.steer_F = h->steer_F;
        ce = launch_prefill(h->weights_view(), h->D, ws, d_x, n, d_out, h->n_sm, st, ev, ids_in, wts_in);
    }
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "forward launch");
}

ds4moe_status ds4moe_forward(ds4moe_t* h, const void* d_x, int32_t n, float* d_out, void* stream) {
    return forward_impl(h, d_x, n, d_out, nullptr, stream, "forward");
}

ds4moe_status ds4moe_forward_routed(ds4moe_t* h, const void* d_x, int32_t n, const int32_t* d_ids, const float* d_w,
                                    float* d_out, void* stream) {
    if (n > 0 && (!d_ids || !d_w)) return fail(DS4MOE_ERR_ARG, "forward_routed: NULL routing");
    if ((reinterpret_cast<uintptr_t>(d_ids) | reinterpret_cast<uintptr_t>(d_w)) & 3)
        return fail(DS4MOE_ERR_ALIGN, "forward_routed: ids and weights must be 4-byte aligned");
    return forward_impl(h, d_x, n, d_out, nullptr, stream, "forward_routed", false, d_ids, d_w);
}

ds4moe_status ds4moe_combine_slots(const float* d_y, const float* d_w, const float* d_base, int32_t n, int32_t k,
                                   int32_t H, float* d_out, void* stream) {
    if (n < 0 || k < 1 || H < 1) return fail(DS4MOE_ERR_ARG, "combine_slots: n %d, k %d, hidden %d", n, k, H);
    if (n == 0) return DS4MOE_OK;
    if (!d_y || !d_w || !d_out) return fail(DS4MOE_ERR_ARG, "combine_slots: NULL buffer");
    const cudaError_t ce = launch_combine_slots(d_y, d_w, d_base, n, k, H, d_out, (cudaStream_t)stream);
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "combine_slots launch");
}

ds4moe_status ds4moe_forward_residual(ds4moe_t* h, const void* d_x, int32_t n, float* d_out, void* stream) {
    return forward_impl(h, d_x, n, d_out, nullptr, stream, "forward_residual", true);
}

ds4moe_status ds4moe_forward_residual_profiled(ds4moe_t* h, const void* d_x, int32_t n, float* d_out,
                                               void* const* events, void* stream) {
    if (!events) return fail(DS4MOE_ERR_ARG, "forward_residual_profiled: NULL events");
    return forward_impl(h, d_x, n, d_out, events, stream, "forward_residual_profiled", true);
}

ds4moe_status ds4moe_forward_chain(ds4moe_t* const* layers, int32_t L, const void* d_x, int32_t n, float* d_out,
                                   float* d_work, void* stream) {
    if (!layers || L < 1) return fail(DS4MOE_ERR_ARG, "forward_chain: no layers");
    if (n == 0) return DS4MOE_OK;
    if (!d_x || !d_out || !d_work) return fail(DS4MOE_ERR_ARG, "forward_chain: NULL buffer");
    if (!aligned16(d_x) || !aligned16(d_out) || !aligned16(d_work))
        return fail(DS4MOE_ERR_ALIGN, "forward_chain: x, out and work must be 16-byte aligned");
    for (int l = 0; l < L; ++l) {
        ds4moe_t* h = layers[l];
        ds4moe_status s = check_forward(h, d_x, n, d_out, "forward_chain");
        if (s != DS4MOE_OK) return s;
        if (n > h->decode_max) return fail(DS4MOE_ERR_ARG, "forward_chain: n_tokens %d above layer %d's decode_max %d", n, l,
                                           h->decode_max);
        if (h->D.H != layers[0]->D.H) return fail(DS4MOE_ERR_SHAPE, "forward_chain: layer %d hidden differs", l);
        if (l > 0 && h->D.act_bf16) return fail(DS4MOE_ERR_SHAPE, "forward_chain: layer %d takes bf16 x", l);
        for (int j = 0; j < l; ++j)
            if (layers[j] == h) return fail(DS4MOE_ERR_ARG, "forward_chain: layer %d repeats layer %d's handle", l, j);
    }
    const size_t H = layers[0]->D.H;
    const size_t xb = (size_t)n * H * (layers[0]->D.act_bf16 ? 2 : 4), ob = (size_t)n * H * 4;
    auto overlap = [](const void* a, size_t na, const void* b, size_t nb) {
        const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
        return x < y + nb && y < x + na;
    };
    if (overlap(d_work, 2 * ob, d_x, xb) || overlap(d_work, 2 * ob, d_out, ob) || overlap(d_x, xb, d_out, ob))
        return fail(DS4MOE_ERR_ARG, "forward_chain: x, out and work overlap");
    cudaStream_t st = (cudaStream_t)stream;
    for (int l = 0; l < L; ++l) {
        ds4moe_t* h = layers[l];
        const void* in = l == 0 ? d_x : d_work + (size_t)((l - 1) % 2) * n * H;
        float* o = l == L - 1 ? d_out : d_work + (size_t)(l % 2) * n * H;
        DecodeWs ws = h->decode_ws();
        ws.xres = in;
        ws.steer_v = h->steer_on ? reinterpret_cast<const float*>(h->weights + h->off_steer) : nullptr;
        ws.steer_F = h->steer_F;
        if (l < L - 1) ws.chain_done = reinterpret_cast<uint32_t*>(h->ws + h->L.hdr) + 10;
        if (l > 0) {
            ds4moe_t* p = layers[l - 1];
            ws.chain_wait = reinterpret_cast<uint32_t*>(p->ws + p->L.hdr) + 10;
            ws.chain_target = decode_combine_ctas(p->D, n, p->steer_on);
        }
        const cudaError_t ce = launch_decode(h->weights_view(), h->D, ws, in, n, o, h->n_sm, st, nullptr);
        if (ce != cudaSuccess) return cuda_fail(ce, "forward_chain launch");
    }
    return DS4MOE_OK;
}

ds4moe_status ds4moe_forward_profiled(ds4moe_t* h, const void* d_x, int32_t n, float* d_out, void* const* events,
                                      void* stream) {
    if (!events) return fail(DS4MOE_ERR_ARG, "forward_profiled: NULL events");
    return forward_impl(h, d_x, n, d_out, events, stream, "forward_profiled");
}

int32_t ds4moe_plan_launches(const ds4moe_t* h, int32_t n) {
    if (!h || n < 1 || n > h->shape.max_tokens) return 0;
    if (n <= h->decode_max) return decode_launches();
    return prefill_launches(h->D);
}

const char* ds4moe_plan_kernel(const ds4moe_t* h, int32_t n, int32_t i) {
    const int nl = ds4moe_plan_launches(h, n);
    if (i < 0 || i >= nl) return nullptr;
    if (h->steer_on && i == nl - 1) return n <= h->decode_max ? "k_combine_steer_decode" : "k_combine_steer_prefill";
    if (n <= h->decode_max) return decode_kernel_name(i);
    return prefill_kernel_name(h->D, i);
}

ds4moe_status ds4moe_forward_host_async(ds4moe_t* h, const void* x_host, int32_t n, float* out_host, void* stream) {
    ds4moe_status s = check_forward(h, x_host, n, out_host, "forward_host_async");
    if (s != DS4MOE_OK) return s;
    if (n == 0) return DS4MOE_OK;
    cudaError_t ce = h->host_streams();
    if (ce != cudaSuccess) return cuda_fail(ce, "forward_host_async: streams");
    cudaStream_t st = (cudaStream_t)stream;
    const int sl = h->slot;
    h->slot ^= 1;
    const size_t xb = (size_t)n * h->D.H * (h->D.act_bf16 ? 2 : 4), ob = (size_t)n * h->D.H * 4;
    void* dx = h->ws + h->L.x_stage + sl * h->L.x_slot;
    float* dout = reinterpret_cast<float*>(h->ws + h->L.out_stage + sl * h->L.out_slot);
    // upload into the slot once the forward that last read it is done
    ce = cudaStreamWaitEvent(h->up, h->ev_done[sl], 0);
    if (ce == cudaSuccess) ce = cudaMemcpyAsync(dx, x_host, xb, cudaMemcpyHostToDevice, h->up);
    if (ce == cudaSuccess) ce = cudaEventRecord(h->ev_in[sl], h->up);
    // the forward once its input has landed and the slot's last result has left
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(st, h->ev_in[sl], 0);
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(st, h->ev_out[sl], 0);
    if (ce != cudaSuccess) return cuda_fail(ce, "forward_host_async: copy in");
    s = ds4moe_forward(h, dx, n, dout, stream);
    if (s != DS4MOE_OK) return s;
    ce = cudaEventRecord(h->ev_done[sl], st);
    // download once the forward is done
    if (ce == cudaSuccess) ce = cudaStreamWaitEvent(h->down, h->ev_done[sl], 0);
    if (ce == cudaSuccess) ce = cudaMemcpyAsync(out_host, dout, ob, cudaMemcpyDeviceToHost, h->down);
    if (ce == cudaSuccess) ce = cudaEventRecord(h->ev_out[sl], h->down);
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "forward_host_async: copy out");
}

ds4moe_status ds4moe_host_sync(ds4moe_t* h) {
    if (!h) return fail(DS4MOE_ERR_ARG, "host_sync: NULL handle");
    if (!h->up) return DS4MOE_OK;
    cudaError_t ce = cudaStreamSynchronize(h->up);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(h->down);   // its copies follow the forwards
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "host_sync");
}

ds4moe_status ds4moe_forward_host(ds4moe_t* h, const void* x_host, int32_t n, float* out_host, void* stream) {
    ds4moe_status s = ds4moe_forward_host_async(h, x_host, n, out_host, stream);
    if (s != DS4MOE_OK) return s;
    if (n == 0) return DS4MOE_OK;
    s = ds4moe_host_sync(h);
    if (s != DS4MOE_OK) return s;
    const cudaError_t ce = cudaStreamSynchronize((cudaStream_t)stream);
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "forward_host: synchronize");
}

ds4moe_status ds4moe_route(ds4moe_t* h, const void* d_x, int32_t n, int32_t* d_ids, float* d_w, void* stream) {
    ds4moe_status s = check_forward(h, d_x, n, d_ids, "route");
    if (s != DS4MOE_OK) return s;
    if (n == 0) return DS4MOE_OK;
    if (!d_w) return fail(DS4MOE_ERR_ARG, "route: NULL weights");
    if (!aligned16(d_x)) return fail(DS4MOE_ERR_ALIGN, "route: x must be 16-byte aligned");
    cudaStream_t st = (cudaStream_t)stream;
    const int32_t* ids_src;
    const float* w_src;
    cudaError_t ce;
    if (n <= h->decode_max) {
        DecodeWs ws = h->decode_ws();
        ce = launch_route(h->weights_view(), h->D, ws, d_x, n, st);
        ids_src = ws.ids;
        w_src = ws.wts;
    } else {
        PrefillWs ws = h->prefill_ws();
        ce = launch_route_prefill(h->weights_view(), h->D, ws, d_x, n, st);
        ids_src = ws.ids;
        w_src = ws.wts;
    }
    if (ce == cudaSuccess)
        ce = cudaMemcpyAsync(d_ids, ids_src, (size_t)n * h->D.k * 4, cudaMemcpyDeviceToDevice, st);
    if (ce == cudaSuccess)
        ce = cudaMemcpyAsync(d_w, w_src, (size_t)n * h->D.k * 4, cudaMemcpyDeviceToDevice, st);
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "route");
}

ds4moe_status ds4moe_probe(ds4moe_t* h, int32_t plan, int32_t which, int32_t e, const void* d_in, int32_t n,
                           float* d_out, void* stream) {
    if (!h) return fail(DS4MOE_ERR_ARG, "probe: NULL handle");
    if (plan != 0 && plan != 1) return fail(DS4MOE_ERR_ARG, "probe: plan %d (0 decode, 1 prefill)", plan);
    if (which != 0 && which != 2) return fail(DS4MOE_ERR_ARG, "probe: which %d (0 gate/up, 2 down)", which);
    if (n < 1 || n > (1 << 20)) return fail(DS4MOE_ERR_ARG, "probe: n_rows %d outside 1..2^20", n);
    if (!d_in || !d_out) return fail(DS4MOE_ERR_ARG, "probe: NULL buffer");
    if (!aligned16(d_in) || !aligned16(d_out)) return fail(DS4MOE_ERR_ALIGN, "probe: buffers must be 16-byte aligned");
    std::string why;
    if (!h->ready(&why)) return fail(DS4MOE_ERR_NOT_READY, "probe: %s", why.c_str());
    if (e < -1 || e >= h->D.E) return fail(DS4MOE_ERR_ARG, "probe: expert %d out of range", e);
    if (e == -1 && !h->shape.has_shared) return fail(DS4MOE_ERR_ARG, "probe: the layer has no shared expert");
    if (plan == 0) {
        if (n > h->decode_max) return fail(DS4MOE_ERR_ARG, "probe: n_rows %d > decode_max %d", n, h->decode_max);
        DecodeWs ws = h->decode_ws();
        ws.probe = e >= 0 ? 1 : 2;
        ws.probe_e = e;
        ws.probe_out = d_out;
        cudaError_t ce = launch_probe_decode(h->weights_view(), h->D, ws, which, d_in, n, h->n_sm, (cudaStream_t)stream);
        return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "probe launch");
    }
    if (h->shape.max_tokens <= h->decode_max)
        return fail(DS4MOE_ERR_NOT_READY, "probe: the prefill plan needs max_tokens > decode_max");
    cudaError_t ce = launch_probe_gemm(h->weights_view(), h->D, h->prefill_ws(), which, e, d_in, n, d_out, h->n_sm,
                                       (cudaStream_t)stream);
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "probe launch");
}

ds4moe_status ds4moe_dequant(ds4moe_t* h, int32_t e, int32_t which, int32_t as_bf16, void* d_out, void* stream) {
    if (!h || !d_out) return fail(DS4MOE_ERR_ARG, "dequant: NULL argument");
    if (!h->weights) return fail(DS4MOE_ERR_NOT_READY, "dequant: buffers not bound");
    cudaStream_t st = (cudaStream_t)stream;
    const int H = h->D.H, I = h->D.I;
    float* of = as_bf16 ? nullptr : (float*)d_out;
    __nv_bfloat16* ob = as_bf16 ? (__nv_bfloat16*)d_out : nullptr;
    const unsigned g = (unsigned)(((int64_t)H * I + 255) / 256);
    if (e == -1) {   // the shared expert (bf16 as stored)
        if (!h->shape.has_shared || !h->shared_set) return fail(DS4MOE_ERR_NOT_READY, "dequant: no shared expert");
        const uint8_t* b = h->weights;
        const __nv_bfloat16* t = reinterpret_cast<const __nv_bfloat16*>(
            b + (which == 0 ? h->off_sh_gate : which == 1 ? h->off_sh_up : h->off_sh_down));
        if (which < 0 || which > 2) return fail(DS4MOE_ERR_ARG, "dequant: which %d", which);
        k_dequant_bf16_tiles<<<g, 256, 0, st>>>(t, which == 2 ? H : I, which == 2 ? I : H, of, ob);
    } else {
        if (e < 0 || e >= h->D.E) return fail(DS4MOE_ERR_ARG, "dequant: expert %d out of range", e);
        if (!h->loaded[e]) return fail(DS4MOE_ERR_NOT_READY, "dequant: expert %d not loaded", e);
        if (h->D.q4) {
            if (which < 0 || which > 2) return fail(DS4MOE_ERR_ARG, "dequant: which %d", which);
            const size_t oq = which == 0 ? h->off_gate_qs : which == 1 ? h->off_up_qs : h->off_down_q;
            const size_t os = which == 0 ? h->off_gate_sc4 : which == 1 ? h->off_up_sc4 : h->off_down_sc4;
            const size_t od = which == 0 ? h->off_gate_dd4 : which == 1 ? h->off_up_dd4 : h->off_down_dd4;
            const int R = which == 2 ? H : I, C = which == 2 ? I : H;
            const unsigned g4 = (unsigned)(((int64_t)R * (C / 64) + 255) / 256);
            k_dequant_q4<<<g4, 256, 0, st>>>(h->weights + oq + e * h->q4_q_stride,
                                             reinterpret_cast<const uint32_t*>(h->weights + os) + e * h->q4_sc_stride,
                                             reinterpret_cast<const uint32_t*>(h->weights + od) + e * h->q4_dd_stride,
                                             R, C, which == 2 ? 1 : 0, of, ob);
        } else if (which == 0 || which == 1) {
            if (!h->grid_set) return fail(DS4MOE_ERR_NOT_READY, "dequant: grid not set");
            const size_t oq = which == 0 ? h->off_gate_qs : h->off_up_qs;
            const size_t od = which == 0 ? h->off_gate_d : h->off_up_d;
            k_dequant_iq2<<<g, 256, 0, st>>>(h->weights + oq + e * h->iq2_qs_stride,
                                             reinterpret_cast<const uint16_t*>(h->weights + od) + e * h->iq2_d_stride,
                                             h->weights + h->off_grid, I, H, of, ob);
        } else if (which == 2) {
            k_dequant_q2<<<g, 256, 0, st>>>(h->weights + h->off_down_q + e * h->q2_q_stride,
                                            reinterpret_cast<const uint32_t*>(h->weights + h->off_down_sc) + e * h->q2_sc_stride,
                                            reinterpret_cast<const uint32_t*>(h->weights + h->off_down_dd) + e * h->q2_dd_stride,
                                            H, I, of, ob);
        } else {
            return fail(DS4MOE_ERR_ARG, "dequant: which %d", which);
        }
    }
    cudaError_t ce = cudaGetLastError();
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "dequant launch");
}

// Device address of the no-allocation scratch on the current device: looked
// up (cudaGetSymbolAddress, with this device current) on the first call per
// device, then cached.  nullptr with *err set on failure.
static float* noalloc_scratch(int dev, cudaError_t* err, bool lookup) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev] && lookup) {
        void* p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (*err != cudaSuccess) return nullptr;
        g_noalloc_addr[dev] = static_cast<float*>(p);
    }
    return g_noalloc_addr[dev];
}

ds4moe_status ds4moe_route_noalloc(ds4moe_t* h, const void* d_x, int32_t n, int32_t* d_ids, float* d_w,
                                   void* stream) {
    // Needs the router and its inputs only: the bound workspace is not used,
    // so a handle bound to a weight buffer (and any workspace) with grid and
    // router loaded is enough.
    if (!h) return fail(DS4MOE_ERR_ARG, "route_noalloc: NULL handle");
    if (n < 0 || n > h->shape.max_tokens)
        return fail(DS4MOE_ERR_ARG, "route_noalloc: n_tokens %d outside 0..%d", n, h->shape.max_tokens);
    if (n == 0) return DS4MOE_OK;
    if (!d_x || !d_ids || !d_w) return fail(DS4MOE_ERR_ARG, "route_noalloc: NULL buffer");
    if (!h->weights) return fail(DS4MOE_ERR_NOT_READY, "route_noalloc: buffers not bound");
    if ((!h->grid_set && !h->D.q4) || !h->router_set)
        return fail(DS4MOE_ERR_NOT_READY, "route_noalloc: router not loaded");
    if (!aligned16(d_x)) return fail(DS4MOE_ERR_ALIGN, "route_noalloc: x must be 16-byte aligned");
    if (n > h->decode_max) return fail(DS4MOE_ERR_ARG, "route_noalloc: n_tokens %d > decode_max %d", n, h->decode_max);
    if ((int64_t)n * h->D.E > kNoAllocLogits)
        return fail(DS4MOE_ERR_ARG, "route_noalloc: n_tokens * n_experts = %lld exceeds the static scratch limit %d",
                    (long long)n * h->D.E, kNoAllocLogits);
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return cuda_fail(ce, "route_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kNoAllocDevices)
        return fail(DS4MOE_ERR_ARG, "route_noalloc: device %d beyond %d", dev, kNoAllocDevices);
    float* base = noalloc_scratch(dev, &ce, true);
    if (!base) return cuda_fail(ce, "route_noalloc: cudaGetSymbolAddress");
    cudaStream_t st = (cudaStream_t)stream;
    // the counters must start at zero (the previous call's are stale); the
    // error word (word 0) stays until ds4moe_get_device_error reads it
    ce = cudaMemsetAsync(base + 1, 0, (kNoAllocHeader - 1) * sizeof(float), st);
    if (ce != cudaSuccess) return cuda_fail(ce, "route_noalloc: clear counters");
    uint32_t* hdr = reinterpret_cast<uint32_t*>(base);
    DecodeWs ws{};
    ws.err = hdr + 0;
    ws.ticket = hdr + 1;
    ws.queue = hdr + 2;
    ws.queue_rt = hdr + 3;
    ws.logits = base + kNoAllocHeader;
    ws.ids = d_ids;
    ws.wts = d_w;
    ce = launch_route(h->weights_view(), h->D, ws, d_x, n, st);
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "route_noalloc launch");
}

ds4moe_status ds4moe_permutation(ds4moe_t* h, const int32_t* d_ids, int32_t n, int32_t* d_counts,
                                 int32_t* d_offsets, int32_t* d_pos_of_slot, void* stream) {
    if (!h) return fail(DS4MOE_ERR_ARG, "permutation: NULL handle");
    if (!d_ids || !d_counts || !d_offsets || !d_pos_of_slot) return fail(DS4MOE_ERR_ARG, "permutation: NULL buffer");
    if (!h->ws) return fail(DS4MOE_ERR_NOT_READY, "permutation: workspace not bound");
    if (h->shape.max_tokens <= h->decode_max)
        return fail(DS4MOE_ERR_NOT_READY, "permutation: the prefill plan needs max_tokens > decode_max");
    if (n < 1 || n > h->shape.max_tokens)
        return fail(DS4MOE_ERR_ARG, "permutation: n_tokens %d outside 1..%d", n, h->shape.max_tokens);
    cudaStream_t st = (cudaStream_t)stream;
    PrefillWs ws = h->prefill_ws();
    cudaError_t ce = launch_permutation(h->D, ws, d_ids, n, st);
    const size_t E = h->D.E, nk = (size_t)n * h->D.k;
    if (ce == cudaSuccess) ce = cudaMemcpyAsync(d_counts, ws.counts, E * 4, cudaMemcpyDeviceToDevice, st);
    if (ce == cudaSuccess) ce = cudaMemcpyAsync(d_offsets, ws.offs, (E + 1) * 4, cudaMemcpyDeviceToDevice, st);
    if (ce == cudaSuccess) ce = cudaMemcpyAsync(d_pos_of_slot, ws.pos_of_slot, nk * 4, cudaMemcpyDeviceToDevice, st);
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "permutation");
}

ds4moe_status ds4moe_selftest_wait(ds4moe_t* h, void* stream) {
    if (!h) return fail(DS4MOE_ERR_ARG, "selftest_wait: NULL handle");
    if (!h->ws) return fail(DS4MOE_ERR_NOT_READY, "selftest_wait: workspace not bound");
    cudaError_t ce = launch_wait_selftest(reinterpret_cast<uint32_t*>(h->ws + h->L.hdr), (cudaStream_t)stream);
    return ce == cudaSuccess ? DS4MOE_OK : cuda_fail(ce, "selftest_wait launch");
}

ds4moe_status ds4moe_get_device_error(ds4moe_t* h, void* stream, int32_t* code) {
    if (!h || !code) return fail(DS4MOE_ERR_ARG, "get_device_error: NULL argument");
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return cuda_fail(ce, "get_device_error: cudaGetDevice");
    // the no-allocation routing's error word on this device, if that entry point has run here
    uint32_t* na = nullptr;
    if (dev >= 0 && dev < kNoAllocDevices) na = reinterpret_cast<uint32_t*>(noalloc_scratch(dev, &ce, false));
    if (!h->ws && !na) return fail(DS4MOE_ERR_NOT_READY, "get_device_error: buffers not bound");
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t v = 0, w = 0;
    ce = cudaStreamSynchronize(st);
    if (ce == cudaSuccess && h->ws) ce = cudaMemcpy(&v, h->ws + h->L.hdr, 4, cudaMemcpyDeviceToHost);
    if (ce == cudaSuccess && v) ce = cudaMemset(h->ws + h->L.hdr, 0, 4);
    if (ce == cudaSuccess && na) ce = cudaMemcpy(&w, na, 4, cudaMemcpyDeviceToHost);
    if (ce == cudaSuccess && w) ce = cudaMemset(na, 0, 4);
    if (ce != cudaSuccess) return cuda_fail(ce, "get_device_error");
    v |= w;
    *code = (int32_t)v;
    if (v & kErrTimeout) return fail(DS4MOE_ERR_TIMEOUT, "a bounded device wait timed out (code %u)", v);
    if (v) return fail(DS4MOE_ERR_DEVICE, "device-side check failed (code %u)", v);
    return DS4MOE_OK;
}

}  // extern "C"
