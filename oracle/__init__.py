"""CPU oracle for the ds4 routed-MoE expert FFN (ctypes wrapper around ds4_oracle.c).

TEST INFRASTRUCTURE ONLY.  The oracle is the slow, plain reference the CUDA
path is checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The library package never imports it and shares no code with it.

Every function takes and returns numpy arrays; the arithmetic is all in
``ds4_oracle.c`` (see its header for the readings each function follows).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ds4_oracle.c")
_LIB = os.path.join(_HERE, "libds4oracle.so")
_lib = None

QK = 256
Q2_BYTES = 84
IQ2_BYTES = 66
Q4_BYTES = 144


def build(force: bool = False) -> str:
    """Compile ds4_oracle.c into libds4oracle.so next to it (gcc, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Layer(ctypes.Structure):
    _fields_ = [
        ("H", ctypes.c_int32), ("I", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
        ("W_r", ctypes.c_void_p), ("b_r", ctypes.c_void_p), ("grid", ctypes.c_void_p),
        ("gate", ctypes.POINTER(ctypes.c_void_p)), ("up", ctypes.POINTER(ctypes.c_void_p)),
        ("down", ctypes.POINTER(ctypes.c_void_p)),
        ("sh_gate", ctypes.c_void_p), ("sh_up", ctypes.c_void_p), ("sh_down", ctypes.c_void_p),
        ("expert_bits", ctypes.c_int32),
    ]


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        L.orc_half_to_double.argtypes = [ctypes.c_uint16]
        L.orc_half_to_double.restype = ctypes.c_double
        L.orc_double_to_half.argtypes = [ctypes.c_double]
        L.orc_double_to_half.restype = ctypes.c_uint16
        L.orc_bf16_round.argtypes = [ctypes.c_float]
        L.orc_bf16_round.restype = ctypes.c_float
        L.orc_bf16_round_array.argtypes = [vp, i64, vp]
        L.orc_dequant_q2k.argtypes = [vp, i64, vp]
        L.orc_dequant_iq2xxs.argtypes = [vp, i64, vp, vp]
        L.orc_pack_q2k.argtypes = [vp, i64, vp]
        L.orc_pack_q2k.restype = ctypes.c_int
        L.orc_dequant_q4k.argtypes = [vp, i64, vp]
        L.orc_pack_q4k.argtypes = [vp, i64, vp]
        L.orc_pack_q4k.restype = ctypes.c_int
        L.orc_pack_iq2xxs.argtypes = [vp, i64, vp, vp]
        L.orc_pack_iq2xxs.restype = ctypes.c_int
        L.orc_router_logit.argtypes = [vp, vp, i32, vp]
        L.orc_router_logit.restype = ctypes.c_float
        L.orc_router_logits.argtypes = [vp, vp, vp, i64, i32, i32, vp]
        L.orc_router_logits_f64.argtypes = [vp, vp, vp, i64, i32, i32, vp]
        L.orc_topk_softmax.argtypes = [vp, i64, i32, i32, vp, vp]
        L.orc_moe_forward.argtypes = [ctypes.POINTER(Layer), vp, i64, i32, vp, vp, vp]
        L.orc_moe_forward.restype = ctypes.c_int
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- scalars
def half_to_double(bits: int) -> float:
    return lib().orc_half_to_double(int(bits))


def double_to_half(v: float) -> int:
    return int(lib().orc_double_to_half(float(v)))


def bf16_round(v) -> np.ndarray:
    """Elementwise bfloat16 round-half-to-even of binary32 values (returned as float32)."""
    a = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.empty_like(a)
    lib().orc_bf16_round_array(_p(a), a.size, _p(out))
    return out.reshape(np.shape(v))


# ---------------------------------------------------------------- formats
def dequant_q2k(blocks: np.ndarray) -> np.ndarray:
    b = _c(blocks, np.uint8).reshape(-1, Q2_BYTES)
    out = np.empty(b.shape[0] * QK, dtype=np.float32)
    lib().orc_dequant_q2k(_p(b), b.shape[0], _p(out))
    return out


def dequant_iq2xxs(blocks: np.ndarray, grid: np.ndarray) -> np.ndarray:
    b = _c(blocks, np.uint8).reshape(-1, IQ2_BYTES)
    g = _c(grid, np.uint8).reshape(256 * 8)
    out = np.empty(b.shape[0] * QK, dtype=np.float32)
    lib().orc_dequant_iq2xxs(_p(b), b.shape[0], _p(g), _p(out))
    return out


def pack_q2k(w: np.ndarray) -> np.ndarray:
    x = _c(w, np.float32).ravel()
    out = np.zeros((x.size // QK, Q2_BYTES), dtype=np.uint8)
    if lib().orc_pack_q2k(_p(x), x.size, _p(out)) != 0:
        raise ValueError("pack_q2k: size must be a multiple of 256")
    return out


def dequant_q4k(blocks: np.ndarray) -> np.ndarray:
    """Q4_K-style blocks (144 bytes / 256 weights, the 4-bit expert variant) -> binary32."""
    b = _c(blocks, np.uint8).reshape(-1, Q4_BYTES)
    out = np.empty(b.shape[0] * QK, dtype=np.float32)
    lib().orc_dequant_q4k(_p(b), b.shape[0], _p(out))
    return out


def pack_q4k(w: np.ndarray) -> np.ndarray:
    x = _c(w, np.float32).ravel()
    out = np.zeros((x.size // QK, Q4_BYTES), dtype=np.uint8)
    if lib().orc_pack_q4k(_p(x), x.size, _p(out)) != 0:
        raise ValueError("pack_q4k: size must be a multiple of 256")
    return out


def pack_iq2xxs(w: np.ndarray, grid: np.ndarray) -> np.ndarray:
    x = _c(w, np.float32).ravel()
    g = _c(grid, np.uint8).reshape(256 * 8)
    out = np.zeros((x.size // QK, IQ2_BYTES), dtype=np.uint8)
    if lib().orc_pack_iq2xxs(_p(x), x.size, _p(g), _p(out)) != 0:
        raise ValueError("pack_iq2xxs: size must be a multiple of 256")
    return out


# ---------------------------------------------------------------- router
def router_logits(x: np.ndarray, W: np.ndarray, b: np.ndarray | None = None) -> np.ndarray:
    x = _c(x, np.float32)
    W = _c(W, np.float32)
    b = _c(b, np.float32)
    n, H = x.shape
    E = W.shape[0]
    out = np.empty((n, E), dtype=np.float32)
    lib().orc_router_logits(_p(x), _p(W), _p(b), n, E, H, _p(out))
    return out


def router_logits_f64(x: np.ndarray, W: np.ndarray, b: np.ndarray | None = None) -> np.ndarray:
    x = _c(x, np.float32)
    W = _c(W, np.float32)
    b = _c(b, np.float32)
    n, H = x.shape
    E = W.shape[0]
    out = np.empty((n, E), dtype=np.float64)
    lib().orc_router_logits_f64(_p(x), _p(W), _p(b), n, E, H, _p(out))
    return out


def topk_softmax(logits: np.ndarray, k: int):
    lg = _c(logits, np.float32)
    n, E = lg.shape
    ids = np.empty((n, k), dtype=np.int32)
    w = np.empty((n, k), dtype=np.float64)
    lib().orc_topk_softmax(_p(lg), n, E, k, _p(ids), _p(w))
    return ids, w


# ---------------------------------------------------------------- layer
def moe_forward(layer: dict, x: np.ndarray, mode: int = 0):
    """Forward of one MoE layer on x [n, H] (float32 values).

    ``layer`` holds: H, I, E, k, W_r [E,H] f32, b_r [E] f32 or None, grid
    [256,8] u8, gate/up/down: sequences of E canonical block arrays (an entry
    may be None for an expert no token selects), sh_gate/sh_up/sh_down: bf16
    bit patterns as uint16 arrays or None; expert_bits (default 2): 2 for
    IQ2_XXS-style gate/up and Q2_K-style down blocks, 4 for Q4_K-style blocks
    in all three.
    mode 0: fp64 decode reading; mode 1: bf16 tensor-core reading.
    Returns (out [n,H] f64, ids [n,k] i32, w [n,k] f64).
    """
    H, I, E, k = (int(layer[s]) for s in ("H", "I", "E", "k"))
    x = _c(x, np.float32).reshape(-1, H)
    n = x.shape[0]
    keep = []

    def arr(a, dt):
        if a is None:
            return None
        c = _c(a, dt)
        keep.append(c)
        return c

    def ptrs(seq):
        vals = []
        for a in seq:
            c = arr(a, np.uint8)
            vals.append(None if c is None else c.ctypes.data)
        return (ctypes.c_void_p * E)(*vals)

    W_r = arr(layer["W_r"], np.float32)
    b_r = arr(layer.get("b_r"), np.float32)
    grid = arr(layer["grid"], np.uint8)
    gate, up, down = ptrs(layer["gate"]), ptrs(layer["up"]), ptrs(layer["down"])
    sg, su, sd = (arr(layer.get(s), np.uint16) for s in ("sh_gate", "sh_up", "sh_down"))
    L = Layer(H, I, E, k, _p(W_r), _p(b_r), _p(grid),
              ctypes.cast(gate, ctypes.POINTER(ctypes.c_void_p)),
              ctypes.cast(up, ctypes.POINTER(ctypes.c_void_p)),
              ctypes.cast(down, ctypes.POINTER(ctypes.c_void_p)),
              _p(sg), _p(su), _p(sd), int(layer.get("expert_bits", 2)))
    out = np.zeros((n, H), dtype=np.float64)
    ids = np.zeros((n, k), dtype=np.int32)
    w = np.zeros((n, k), dtype=np.float64)
    rc = lib().orc_moe_forward(ctypes.byref(L), _p(x), n, int(mode), _p(out), _p(ids), _p(w))
    if rc != 0:
        raise ValueError("orc_moe_forward: bad argument or missing expert blocks")
    return out, ids, w


def steer(y: np.ndarray, v: np.ndarray, F: float) -> np.ndarray:
    """Directional steering of a layer output, per token: y - F v (v . y), in fp64.

    Follows the pages' server option for steering after the FFN outputs, one
    binary32 direction vector per layer (the server's option list in the
    modu-print.com article on ds4.c).
    """
    y = np.asarray(y, dtype=np.float64)
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    return y - float(F) * np.outer(y @ v, v)


def chain_forward(layers, x: np.ndarray, mode: int = 0):
    """A chain of layers with the residual step x_{l+1} = x_l + MoE_l(x_l).

    Follows the pages' multi-token-prediction draft-and-verify (the server's
    option list in the modu-print.com article on ds4.c; the MTP note in the
    amuse.peoplentools.com summary) as read for a stack of MoE layers with no
    norm in between.  Each layer's input is binary32
    (the decode plan's activation type): the fp64 sum is rounded to binary32
    before the next layer.  Returns (x_L as float32 [n,H], per-layer ids,
    per-layer inputs as float32).
    """
    cur = np.asarray(x, dtype=np.float32).reshape(-1, int(layers[0]["H"]))
    ids_all, inputs = [], []
    for lay in layers:
        inputs.append(cur.copy())
        out, ids, _ = moe_forward(lay, cur, mode)
        ids_all.append(ids)
        cur = (cur.astype(np.float64) + out).astype(np.float32)
    return cur, ids_all, inputs


def layer_from_torch(layer: dict, experts=None) -> dict:
    """numpy view of a synthetic layer (torch tensors, any device) for moe_forward.

    `experts` limits which experts' blocks are copied to the host (the others
    stay None); the shared expert's bfloat16 tensors become uint16 bit patterns.
    """
    import torch

    E = int(layer["E"])
    keep = range(E) if experts is None else sorted(set(int(e) for e in experts))
    gate, up, down = [None] * E, [None] * E, [None] * E
    for e in keep:
        gate[e] = layer["gate"][e].cpu().numpy()
        up[e] = layer["up"][e].cpu().numpy()
        down[e] = layer["down"][e].cpu().numpy()
    b = layer.get("b_r")

    def bits(t):
        return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)

    out = dict(H=layer["H"], I=layer["I"], E=E, k=layer["k"], W_r=layer["W_r"].cpu().numpy(),
               b_r=None if b is None else b.cpu().numpy(), grid=layer["grid"].cpu().numpy(),
               gate=gate, up=up, down=down, sh_gate=None, sh_up=None, sh_down=None,
               expert_bits=int(layer.get("expert_bits", 2)))
    if layer.get("sh_gate") is not None:
        out.update(sh_gate=bits(layer["sh_gate"]), sh_up=bits(layer["sh_up"]), sh_down=bits(layer["sh_down"]))
    return out
