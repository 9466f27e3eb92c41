"""Bit-exactness of the weights the hot-path kernels multiply, through the kernels themselves.

ds4moe_probe runs a plan's projection kernels on caller rows routed to one
expert and returns the raw accumulators.  One-hot rows (row c = e_c) give
back column c of each weight matrix exactly as the kernel consumed it: a
single nonzero product with 1.0, added to zeros.  Those columns must equal
the oracle's dequantized weights bit for bit -- rounded to bfloat16 for the
prefill plan (its tensor cores take bf16), binary32 for the decode plan.
Hand-built edge blocks (subnormal and negative scales, zero scales, the
largest group scale, all codes 3, every grid row) are included.
"""
import numpy as np
import pytest
import torch

import bit_quantized_moe_softmax_b200 as m
from bit_quantized_moe_softmax_b200 import synth
from tests._util import pack_with_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_moe_softmax_b200 import build

    build.build()


def _load(L, max_tokens, act=m.DS4MOE_ACT_F32):
    lay = m.MoELayer(L["H"], L["I"], L["E"], L["k"], max_tokens, act_dtype=act,
                     has_shared=L.get("sh_gate") is not None, has_bias=L.get("b_r") is not None)
    lay.load(L)
    return lay


def _probe_columns(lay, plan, which, e):
    """[K][rows]: column c of the probed matrices (gate rows then up rows for which 0).

    The decode plan (plan 0) takes at most decode_max rows per call: the
    one-hot rows go through it eight at a time."""
    K = lay.H if which == 0 else lay.I
    in_dtype = torch.bfloat16 if (plan == 1 or (which == 0 and lay.act_dtype == m.DS4MOE_ACT_BF16)) else torch.float32
    eye = torch.eye(K, device="cuda", dtype=in_dtype)
    out = torch.empty(K, 2 * lay.I if which == 0 else lay.H, dtype=torch.float32, device="cuda")
    step = K if plan == 1 else 8
    for r0 in range(0, K, step):
        m.ds4moe_probe(lay.h, plan, which, e, eye[r0:r0 + step], out[r0:r0 + step])
    torch.cuda.synchronize()
    assert m.ds4moe_get_device_error(lay.h) == 0
    return out.cpu().numpy()


def _ref_columns(orc, L, which, e, bf16):
    H, I = L["H"], L["I"]
    grid = L["grid"].cpu().numpy()
    if e < 0:
        mats = ([L["sh_gate"], L["sh_up"]] if which == 0 else [L["sh_down"]])
        ref = [t.cpu().float().numpy() for t in mats]
    elif which == 0:
        ref = [orc.dequant_iq2xxs(L[n][e].cpu().numpy(), grid).reshape(I, H) for n in ("gate", "up")]
    else:
        ref = [orc.dequant_q2k(L["down"][e].cpu().numpy()).reshape(H, I)]
    ref = np.concatenate(ref, axis=0).T          # [K][rows]
    return orc.bf16_round(ref) if bf16 else ref


def _same_bits(a, b):
    # signed zeros compare equal: a zero weight (d = 0 blocks carry sign bits)
    # reaches the probe's sum as -0 or +0, and -0 + +0 = +0
    a = (np.ascontiguousarray(a, np.float32) + np.float32(0)).view(np.uint32)
    b = (np.ascontiguousarray(b, np.float32) + np.float32(0)).view(np.uint32)
    bad = np.flatnonzero(a != b)
    assert bad.size == 0, "%d words differ, first at %s: %08x vs %08x" % (
        bad.size, np.unravel_index(bad[0], a.shape), a.flat[bad[0]], b.flat[bad[0]])


@pytest.mark.parametrize("plan", [0, 1])
def test_probe_tiny_bit_exact(orc, plan):
    L = synth.float_layer(synth.TINY, 0)
    L.update(pack_with_oracle(orc, L))
    lay = _load(L, max_tokens=64)
    for e in (0, 5, -1):
        for which in (0, 2):
            _same_bits(_probe_columns(lay, plan, which, e), _ref_columns(orc, L, which, e, bf16=plan == 1))


@pytest.mark.parametrize("plan", [0, 1])
def test_probe_full_shape_bit_exact(orc, plan):
    """Full-size matrices (4096 x 2048) of three experts and the shared expert."""
    L = synth.packed_layer(synth.FULL, 31, device="cuda")
    lay = _load(L, max_tokens=16)
    for e in (0, 137, 255, -1):
        for which in (0, 2):
            _same_bits(_probe_columns(lay, plan, which, e), _ref_columns(orc, L, which, e, bf16=plan == 1))


def _edge_layer():
    """A tiny layer (one expert) whose blocks carry the format's edge cases."""
    H, I = 256, 128
    rng = np.random.default_rng(77)
    nb = I * H // 256
    iq = rng.integers(0, 256, (2, nb, 66), dtype=np.uint8)
    q2 = rng.integers(0, 256, (1, nb, 84), dtype=np.uint8)
    half = lambda v: np.frombuffer(np.float16(v).tobytes(), np.uint8)
    iq_d = [6.0e-8, -2.5e-3, 0.0, 65504.0 / 1024, 1.0, -0.125, 2.0 ** -14, 3.1e-3]   # subnormal, negative, zero, ...
    q2_d = [(6.0e-8, 1.2e-7), (-2.0e-3, 3.0e-3), (0.0, 0.0), (1.0, 0.5), (2.5e-3, -1.5e-3), (2.0 ** -24, 0.0),
            (4.0e-3, 4.0e-3), (1e-3, 6.1e-5)]
    for b in range(nb):
        for mat in range(2):
            iq[mat, b, 0:2] = half(iq_d[b % len(iq_d)])
        d, dmin = q2_d[b % len(q2_d)]
        q2[0, b, 80:82] = half(d)
        q2[0, b, 82:84] = half(dmin)
    iq[:, 1, 2 + 8 * np.arange(8) + 7] |= 0xF0      # every group of block 1: s = 15
    q2[0, 3, 16:80] = 0xFF                          # block 3: all codes 3
    q2[0, 3, 0:16] = 0xFF                           # ... with sc = m = 15
    q2[0, 4, 0:16] = 0x00                           # block 4: sc = m = 0
    iq[0, 5, 2:66] = 0                              # block 5: grid row 0, no negatives, s = 0
    grid = synth.grid_table(0)
    for g in range(8):                              # blocks 6..13: all 256 grid rows, once each
        for c in range(4):
            for b in range(8):
                iq[0, 6 + b, 2 + 8 * g + c] = 32 * b + 4 * g + c
    L = dict(H=H, I=I, E=1, k=1, W_r=torch.zeros(1, H), b_r=None, grid=grid,
             gate=torch.from_numpy(iq[0:1].copy()), up=torch.from_numpy(iq[1:2].copy()),
             down=torch.from_numpy(q2.copy()))
    return L


@pytest.mark.parametrize("plan", [0, 1])
def test_probe_edge_blocks_bit_exact(orc, plan):
    L = _edge_layer()
    lay = m.MoELayer(L["H"], L["I"], 1, 1, 64, has_shared=False)
    lay.load(L)
    for which in (0, 2):
        got = _probe_columns(lay, plan, which, 0)
        ref = _ref_columns(orc, L, which, 0, bf16=plan == 1)
        assert np.isfinite(ref).all()
        _same_bits(got, ref)
