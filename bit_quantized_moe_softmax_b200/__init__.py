"""ds4 routed-MoE expert FFN on B200 (sm_100a): Python binding of libds4moe.so.

The functions below carry the names of the C ABI in ``include/ds4moe.h`` and
only marshal arguments: torch tensors become device pointers, the current
torch stream becomes the ``stream`` argument.  Every step of the layer runs in
the library's CUDA kernels; there is no CPU or PyTorch fallback, and loading
fails loudly when the library is missing.

``MoELayer`` is plumbing on top: it allocates the weight and workspace
buffers with torch, binds them and loads a layer.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libds4moe.so")
_lib = None

DS4MOE_ACT_F32 = 0
DS4MOE_ACT_BF16 = 1

STATUS = {0: "OK", -1: "ERR_ARG", -2: "ERR_ALIGN", -3: "ERR_SHAPE", -4: "ERR_NOT_READY", -5: "ERR_CUDA",
          -6: "ERR_TIMEOUT", -7: "ERR_DEVICE"}

# Every symbol include/ds4moe.h declares.
EXPORTS = ("ds4moe_create", "ds4moe_destroy", "ds4moe_weight_bytes", "ds4moe_workspace_bytes", "ds4moe_bind",
           "ds4moe_pack_q2k", "ds4moe_pack_iq2xxs", "ds4moe_set_grid", "ds4moe_set_router", "ds4moe_set_expert",
           "ds4moe_set_shared", "ds4moe_forward", "ds4moe_forward_host", "ds4moe_route", "ds4moe_dequant",
           "ds4moe_get_device_error", "ds4moe_last_error", "ds4moe_plan_launches", "ds4moe_plan_kernel",
           "ds4moe_forward_profiled", "ds4moe_route_noalloc", "ds4moe_forward_residual",
           "ds4moe_forward_residual_profiled", "ds4moe_set_steering", "ds4moe_forward_host_async",
           "ds4moe_host_sync", "ds4moe_probe", "ds4moe_selftest_wait",
           "ds4moe_permutation", "ds4moe_pack_q4k", "ds4moe_forward_chain", "ds4moe_forward_routed",
           "ds4moe_combine_slots")


class ds4moe_shape(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("max_tokens", ctypes.c_int32), ("act_dtype", ctypes.c_int32),
                ("has_shared", ctypes.c_int32), ("has_bias", ctypes.c_int32), ("decode_max", ctypes.c_int32),
                ("expert_bits", ctypes.c_int32)]


class Ds4MoeError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__("%s: %s (%s)" % (where, msg, STATUS.get(status, status)))
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libds4moe.so from the package directory (built by build.py); raise if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libds4moe.so not built: run `python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        sig = {
            "ds4moe_create": ([ctypes.POINTER(ds4moe_shape), ctypes.POINTER(vp)], i32),
            "ds4moe_destroy": ([vp], i32),
            "ds4moe_weight_bytes": ([vp], sz),
            "ds4moe_workspace_bytes": ([vp, i32], sz),
            "ds4moe_bind": ([vp, vp, sz, vp, sz, vp], i32),
            "ds4moe_pack_q2k": ([vp, i64, vp, vp], i32),
            "ds4moe_pack_q4k": ([vp, i64, vp, vp], i32),
            "ds4moe_pack_iq2xxs": ([vp, i64, vp, vp, vp], i32),
            "ds4moe_set_grid": ([vp, vp, vp], i32),
            "ds4moe_set_router": ([vp, vp, vp, vp], i32),
            "ds4moe_set_expert": ([vp, i32, vp, vp, vp, vp], i32),
            "ds4moe_set_shared": ([vp, vp, vp, vp, vp], i32),
            "ds4moe_forward": ([vp, vp, i32, vp, vp], i32),
            "ds4moe_forward_host": ([vp, vp, i32, vp, vp], i32),
            "ds4moe_forward_host_async": ([vp, vp, i32, vp, vp], i32),
            "ds4moe_host_sync": ([vp], i32),
            "ds4moe_route": ([vp, vp, i32, vp, vp, vp], i32),
            "ds4moe_dequant": ([vp, i32, i32, i32, vp, vp], i32),
            "ds4moe_probe": ([vp, i32, i32, i32, vp, i32, vp, vp], i32),
            "ds4moe_selftest_wait": ([vp, vp], i32),
            "ds4moe_permutation": ([vp, vp, i32, vp, vp, vp, vp], i32),
            "ds4moe_get_device_error": ([vp, vp, ctypes.POINTER(i32)], i32),
            "ds4moe_last_error": ([], ctypes.c_char_p),
            "ds4moe_plan_launches": ([vp, i32], i32),
            "ds4moe_plan_kernel": ([vp, i32, i32], ctypes.c_char_p),
            "ds4moe_forward_profiled": ([vp, vp, i32, vp, ctypes.POINTER(vp), vp], i32),
            "ds4moe_route_noalloc": ([vp, vp, i32, vp, vp, vp], i32),
            "ds4moe_forward_residual": ([vp, vp, i32, vp, vp], i32),
            "ds4moe_forward_chain": ([ctypes.POINTER(vp), i32, vp, i32, vp, vp, vp], i32),
            "ds4moe_forward_routed": ([vp, vp, i32, vp, vp, vp, vp], i32),
            "ds4moe_combine_slots": ([vp, vp, vp, i32, i32, i32, vp, vp], i32),
            "ds4moe_set_steering": ([vp, vp, ctypes.c_float, vp], i32),
            "ds4moe_forward_residual_profiled": ([vp, vp, i32, vp, ctypes.POINTER(vp), vp], i32),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def ds4moe_last_error() -> str:
    return lib().ds4moe_last_error().decode()


def _ok(status: int, where: str):
    if status != 0:
        raise Ds4MoeError(status, where, ds4moe_last_error())


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


# ------------------------------------------------------------------ C ABI names
def ds4moe_create(hidden, inter, n_experts, top_k, max_tokens, act_dtype=DS4MOE_ACT_F32, has_shared=1,
                  has_bias=0, decode_max=0, expert_bits=0) -> int:
    s = ds4moe_shape(hidden, inter, n_experts, top_k, max_tokens, act_dtype, has_shared, has_bias, decode_max,
                     expert_bits)
    h = ctypes.c_void_p()
    _ok(lib().ds4moe_create(ctypes.byref(s), ctypes.byref(h)), "ds4moe_create")
    return h.value


def ds4moe_destroy(h: int):
    _ok(lib().ds4moe_destroy(h), "ds4moe_destroy")


def ds4moe_weight_bytes(h: int) -> int:
    return lib().ds4moe_weight_bytes(h)


def ds4moe_workspace_bytes(h: int, n_tokens: int) -> int:
    return lib().ds4moe_workspace_bytes(h, n_tokens)


def ds4moe_bind(h: int, weights: torch.Tensor, workspace: torch.Tensor | None, stream=None):
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _ok(lib().ds4moe_bind(h, _ptr(weights), weights.numel() * weights.element_size(), _ptr(workspace), wsb,
                          _stream(stream)), "ds4moe_bind")


def ds4moe_pack_q2k(w: torch.Tensor, blocks: torch.Tensor, stream=None):
    _ok(lib().ds4moe_pack_q2k(_ptr(w), w.numel(), _ptr(blocks), _stream(stream)), "ds4moe_pack_q2k")


def ds4moe_pack_q4k(w: torch.Tensor, blocks: torch.Tensor, stream=None):
    _ok(lib().ds4moe_pack_q4k(_ptr(w), w.numel(), _ptr(blocks), _stream(stream)), "ds4moe_pack_q4k")


def ds4moe_pack_iq2xxs(w: torch.Tensor, grid: torch.Tensor, blocks: torch.Tensor, stream=None):
    _ok(lib().ds4moe_pack_iq2xxs(_ptr(w), w.numel(), _ptr(grid), _ptr(blocks), _stream(stream)),
        "ds4moe_pack_iq2xxs")


def ds4moe_set_grid(h: int, grid: torch.Tensor, stream=None):
    _ok(lib().ds4moe_set_grid(h, _ptr(grid), _stream(stream)), "ds4moe_set_grid")


def ds4moe_set_router(h: int, W: torch.Tensor, bias: torch.Tensor | None = None, stream=None):
    _ok(lib().ds4moe_set_router(h, _ptr(W), _ptr(bias), _stream(stream)), "ds4moe_set_router")


def ds4moe_set_expert(h: int, e: int, gate: torch.Tensor, up: torch.Tensor, down: torch.Tensor, stream=None):
    _ok(lib().ds4moe_set_expert(h, e, _ptr(gate), _ptr(up), _ptr(down), _stream(stream)), "ds4moe_set_expert")


def ds4moe_set_shared(h: int, gate: torch.Tensor, up: torch.Tensor, down: torch.Tensor, stream=None):
    _ok(lib().ds4moe_set_shared(h, _ptr(gate), _ptr(up), _ptr(down), _stream(stream)), "ds4moe_set_shared")


def ds4moe_forward(h: int, x: torch.Tensor, out: torch.Tensor, stream=None):
    _ok(lib().ds4moe_forward(h, _ptr(x), x.shape[0], _ptr(out), _stream(stream)), "ds4moe_forward")


def ds4moe_set_steering(h: int, v: torch.Tensor | None, F: float, stream=None):
    _ok(lib().ds4moe_set_steering(h, None if v is None else _ptr(v), ctypes.c_float(F), _stream(stream)),
        "ds4moe_set_steering")


def ds4moe_forward_routed(h: int, x: torch.Tensor, ids: torch.Tensor, w: torch.Tensor, out: torch.Tensor,
                          stream=None):
    _ok(lib().ds4moe_forward_routed(h, _ptr(x), x.shape[0], _ptr(ids), _ptr(w), _ptr(out), _stream(stream)),
        "ds4moe_forward_routed")


def ds4moe_combine_slots(y: torch.Tensor, w: torch.Tensor, base: torch.Tensor | None, out: torch.Tensor,
                         stream=None):
    n, k = w.shape
    _ok(lib().ds4moe_combine_slots(_ptr(y), _ptr(w), _ptr(base), n, k, out.shape[1], _ptr(out), _stream(stream)),
        "ds4moe_combine_slots")


def ds4moe_forward_chain(handles, x: torch.Tensor, out: torch.Tensor, work: torch.Tensor, stream=None):
    arr = (ctypes.c_void_p * len(handles))(*handles)
    _ok(lib().ds4moe_forward_chain(arr, len(handles), _ptr(x), x.shape[0], _ptr(out), _ptr(work), _stream(stream)),
        "ds4moe_forward_chain")


def ds4moe_forward_residual(h: int, x: torch.Tensor, out: torch.Tensor, stream=None):
    _ok(lib().ds4moe_forward_residual(h, _ptr(x), x.shape[0], _ptr(out), _stream(stream)), "ds4moe_forward_residual")


def ds4moe_forward_residual_profiled(h: int, x: torch.Tensor, out: torch.Tensor, events, stream=None):
    arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    _ok(lib().ds4moe_forward_residual_profiled(h, _ptr(x), x.shape[0], _ptr(out), arr, _stream(stream)),
        "ds4moe_forward_residual_profiled")


def ds4moe_plan_launches(h: int, n_tokens: int) -> int:
    return lib().ds4moe_plan_launches(h, n_tokens)


def ds4moe_plan_kernel(h: int, n_tokens: int, i: int) -> str | None:
    r = lib().ds4moe_plan_kernel(h, n_tokens, i)
    return None if r is None else r.decode()


def ds4moe_forward_profiled(h: int, x: torch.Tensor, out: torch.Tensor, events, stream=None):
    """events: a flat list of torch.cuda.Event(enable_timing=True), 2 per launch of the plan."""
    arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    _ok(lib().ds4moe_forward_profiled(h, _ptr(x), x.shape[0], _ptr(out), arr, _stream(stream)),
        "ds4moe_forward_profiled")


def ds4moe_forward_host(h: int, x_host: torch.Tensor, out_host: torch.Tensor, stream=None):
    _ok(lib().ds4moe_forward_host(h, _ptr(x_host), x_host.shape[0], _ptr(out_host), _stream(stream)),
        "ds4moe_forward_host")


def ds4moe_forward_host_async(h: int, x_host: torch.Tensor, out_host: torch.Tensor, stream=None):
    """Enqueue a host-buffer forward; out_host is valid after ds4moe_host_sync(h)."""
    _ok(lib().ds4moe_forward_host_async(h, _ptr(x_host), x_host.shape[0], _ptr(out_host), _stream(stream)),
        "ds4moe_forward_host_async")


def ds4moe_host_sync(h: int):
    _ok(lib().ds4moe_host_sync(h), "ds4moe_host_sync")


def ds4moe_route(h: int, x: torch.Tensor, ids: torch.Tensor, w: torch.Tensor, stream=None):
    _ok(lib().ds4moe_route(h, _ptr(x), x.shape[0], _ptr(ids), _ptr(w), _stream(stream)), "ds4moe_route")


def ds4moe_route_noalloc(h: int, x: torch.Tensor, ids: torch.Tensor, w: torch.Tensor, stream=None):
    """Routing with the library's static device scratch instead of the bound workspace.

    For callers that cannot allocate device memory (a host that owns every
    device buffer through its own pool, or code that must not stall the device
    with a synchronizing allocation); the handle needs only its weight buffer
    bound.  Limit: n_tokens * n_experts <= 8192; calls that overlap on the GPU
    race on the shared scratch.
    """
    _ok(lib().ds4moe_route_noalloc(h, _ptr(x), x.shape[0], _ptr(ids), _ptr(w), _stream(stream)),
        "ds4moe_route_noalloc")


def ds4moe_probe(h: int, plan: int, which: int, e: int, inp: torch.Tensor, out: torch.Tensor, stream=None):
    """Raw accumulators of one plan's projection kernels on caller rows, all routed to expert e (-1: shared)."""
    _ok(lib().ds4moe_probe(h, plan, which, e, _ptr(inp), inp.shape[0], _ptr(out), _stream(stream)), "ds4moe_probe")


def ds4moe_dequant(h: int, e: int, which: int, as_bf16: int, out: torch.Tensor, stream=None):
    _ok(lib().ds4moe_dequant(h, e, which, as_bf16, _ptr(out), _stream(stream)), "ds4moe_dequant")


def ds4moe_permutation(h: int, ids: torch.Tensor, counts: torch.Tensor, offsets: torch.Tensor,
                       pos_of_slot: torch.Tensor, stream=None):
    """The prefill plan's stable counting sort of the (token, slot) pairs of ids [n][k] by expert."""
    _ok(lib().ds4moe_permutation(h, _ptr(ids), ids.shape[0], _ptr(counts), _ptr(offsets), _ptr(pos_of_slot),
                                 _stream(stream)), "ds4moe_permutation")


def ds4moe_selftest_wait(h: int, stream=None):
    """A bounded wait on an mbarrier nothing arrives at: gives up after its limit and sets error bit 1."""
    _ok(lib().ds4moe_selftest_wait(h, _stream(stream)), "ds4moe_selftest_wait")


def ds4moe_get_device_error(h: int, stream=None) -> int:
    code = ctypes.c_int32(0)
    st = lib().ds4moe_get_device_error(h, _stream(stream), ctypes.byref(code))
    if st not in (0, -6, -7):
        _ok(st, "ds4moe_get_device_error")
    return code.value


# ------------------------------------------------------------------ plumbing
class MoELayer:
    """One layer's handle plus torch-allocated weight and workspace buffers.

    ``load`` takes a dict with H, I, E, k, W_r, b_r, grid and either packed
    blocks (gate, up: [E, I*H/256, 66] u8; down: [E, H*I/256, 84] u8) or float
    weights to pack on the device (gate_f, up_f: [E, I, H]; down_f: [E, H, I]),
    plus sh_gate/sh_up/sh_down bf16 when has_shared.  With expert_bits=4 all
    three expert matrices are Q4_K-style blocks ([E, n/256, 144] u8) and no
    grid is needed.
    """

    def __init__(self, H, I, E, k, max_tokens, act_dtype=DS4MOE_ACT_F32, has_shared=True, has_bias=False,
                 decode_max=0, device="cuda", expert_bits=0):
        self.H, self.I, self.E, self.k = H, I, E, k
        self.expert_bits = expert_bits
        self.max_tokens = max_tokens
        self.act_dtype = act_dtype
        self.device = torch.device(device)
        self.h = ds4moe_create(H, I, E, k, max_tokens, act_dtype, int(has_shared), int(has_bias), decode_max,
                               expert_bits)
        wb = ds4moe_weight_bytes(self.h)
        sb = ds4moe_workspace_bytes(self.h, max_tokens)
        self.weights = torch.empty(wb, dtype=torch.uint8, device=self.device)
        self.workspace = torch.empty(sb, dtype=torch.uint8, device=self.device)
        ds4moe_bind(self.h, self.weights, self.workspace)

    def __del__(self):
        h = getattr(self, "h", None)
        if h:
            try:
                ds4moe_destroy(h)
            except Exception:
                pass
            self.h = None

    def pack(self, layer: dict) -> dict:
        """Pack float expert weights with the device quantizers; returns gate/up/down blocks."""
        H, I, E = self.H, self.I, self.E
        dev = self.device
        nb = I * H // 256
        if self.expert_bits == 4:
            blocks = {}
            for name in ("gate", "up", "down"):
                t = torch.empty(E, nb, 144, dtype=torch.uint8, device=dev)
                for e in range(E):
                    ds4moe_pack_q4k(layer[name + "_f"][e].to(dev).contiguous(), t[e])
                blocks[name] = t
            return blocks
        grid = layer["grid"].to(dev).contiguous()
        gate = torch.empty(E, nb, 66, dtype=torch.uint8, device=dev)
        up = torch.empty(E, nb, 66, dtype=torch.uint8, device=dev)
        down = torch.empty(E, nb, 84, dtype=torch.uint8, device=dev)
        for e in range(E):
            ds4moe_pack_iq2xxs(layer["gate_f"][e].to(dev).contiguous(), grid, gate[e])
            ds4moe_pack_iq2xxs(layer["up_f"][e].to(dev).contiguous(), grid, up[e])
            ds4moe_pack_q2k(layer["down_f"][e].to(dev).contiguous(), down[e])
        return dict(gate=gate, up=up, down=down)

    def load(self, layer: dict):
        dev = self.device
        if "gate" not in layer:
            layer = {**layer, **self.pack(layer)}
        if layer.get("grid") is not None:
            ds4moe_set_grid(self.h, layer["grid"].to(dev).contiguous())
        b = layer.get("b_r")
        ds4moe_set_router(self.h, layer["W_r"].to(dev).contiguous(), None if b is None else b.to(dev).contiguous())
        for e in range(self.E):
            ds4moe_set_expert(self.h, e, layer["gate"][e].to(dev).contiguous(), layer["up"][e].to(dev).contiguous(),
                              layer["down"][e].to(dev).contiguous())
        if layer.get("sh_gate") is not None:
            ds4moe_set_shared(self.h, layer["sh_gate"].to(dev).contiguous(), layer["sh_up"].to(dev).contiguous(),
                              layer["sh_down"].to(dev).contiguous())
        torch.cuda.current_stream(dev).synchronize()
        return layer

    def forward(self, x: torch.Tensor, out: torch.Tensor | None = None, residual: bool = False) -> torch.Tensor:
        """The layer on x; with residual=True, x + the layer (x and out must not overlap)."""
        if out is None:
            out = torch.empty(x.shape[0], self.H, dtype=torch.float32, device=x.device)
        (ds4moe_forward_residual if residual else ds4moe_forward)(self.h, x, out)
        return out

    def set_steering(self, v: torch.Tensor | None, F: float = 1.0):
        """Steer the layer output: y -= F v (v . y) (v: [H] binary32 on the device; None turns it off)."""
        ds4moe_set_steering(self.h, v, F)

    def route(self, x: torch.Tensor):
        ids = torch.empty(x.shape[0], self.k, dtype=torch.int32, device=x.device)
        w = torch.empty(x.shape[0], self.k, dtype=torch.float32, device=x.device)
        ds4moe_route(self.h, x, ids, w)
        return ids, w

    def dequant(self, e: int, which: int, as_bf16: bool = False) -> torch.Tensor:
        rows, cols = (self.H, self.I) if which == 2 else (self.I, self.H)
        out = torch.empty(rows, cols, dtype=torch.bfloat16 if as_bf16 else torch.float32, device=self.device)
        ds4moe_dequant(self.h, e, which, int(as_bf16), out)
        return out
