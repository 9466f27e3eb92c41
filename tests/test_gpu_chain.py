"""GPU parity of chained layers (the residual step x_{l+1} = x_l + MoE_l(x_l)) against the CPU oracle.

The multi-token-prediction verify workload: 8 chained layers, router logits
N(0,1) (W_r ~ N(0, 1/H)), 2 tokens per step and a sweep of 1/2/4/8.  Per
layer the oracle gets the GPU's own layer input, so routing ids are compared
exactly; the final output is compared with the oracle's independent chain.
Bars: decode plan 1e-4 of max|ref|, prefill plan 2e-3 (bf16 reading).
"""
import math

import numpy as np
import pytest
import torch

import bit_quantized_moe_softmax_b200 as m
from bit_quantized_moe_softmax_b200 import synth
from tests._util import oracle_layer, pack_with_oracle, rel_err

pytestmark = pytest.mark.gpu

LAYERS = 8


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_moe_softmax_b200 import build

    build.build()


def _tiny_chain(orc, act=m.DS4MOE_ACT_F32, max_tokens=8):
    H = 256
    Ls, lays = [], []
    for l in range(LAYERS):
        L = synth.float_layer(synth.Shape(H=H, I=128, E=8, k=2), 100 + l, router_std=1.0 / math.sqrt(H))
        L.update(pack_with_oracle(orc, L))
        lay = m.MoELayer(H, 128, 8, 2, max_tokens, act_dtype=act)
        lay.load(L)
        Ls.append(L)
        lays.append(lay)
    return Ls, lays


def _run_chain(lays, x):
    """GPU chain; returns every layer's input and the final output (device tensors)."""
    inputs, cur = [], x
    for lay in lays:
        inputs.append(cur)
        cur = lay.forward(cur, residual=True)
    return inputs, cur


@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_chain_tiny_decode(orc, n):
    Ls, lays = _tiny_chain(orc)
    x = synth.tokens(n, 256, seed=20 + n).cuda()
    inputs, out = _run_chain(lays, x)
    for L, lay, xin in zip(Ls, lays, inputs):
        ids, _ = lay.route(xin)
        xl = xin.cpu().numpy()
        ref, rid, _ = orc.moe_forward(oracle_layer(L), xl)
        assert np.array_equal(ids.cpu().numpy(), rid)
    ref_final, _, _ = orc.chain_forward([oracle_layer(L) for L in Ls], x.cpu().numpy())
    assert rel_err(out.cpu().numpy(), ref_final) < 1e-4


def test_chain_layer_residual_is_x_plus_layer(orc):
    Ls, lays = _tiny_chain(orc)
    x = synth.tokens(4, 256, seed=3).cuda()
    y = lays[0].forward(x)
    r = lays[0].forward(x, residual=True)
    assert torch.equal(r, x + y)


def test_chain_rejects_overlap(orc):
    Ls, lays = _tiny_chain(orc)
    buf = torch.zeros(8, 256, device="cuda")
    with pytest.raises(m.Ds4MoeError):
        m.ds4moe_forward_residual(lays[0].h, buf[:4], buf[2:6])


def test_chain_tiny_prefill(orc):
    """The residual step through the tensor-core plan (64 bf16 tokens per layer, 3 layers)."""
    Ls, lays = _tiny_chain(orc, act=m.DS4MOE_ACT_F32, max_tokens=64)
    x = synth.tokens(64, 256, seed=9).cuda()
    cur = x
    for L, lay in zip(Ls[:3], lays[:3]):
        nxt = lay.forward(cur, residual=True)
        ref, _, _ = orc.moe_forward(oracle_layer(L), cur.cpu().numpy(), mode=1)
        got = (nxt - cur).cpu().numpy()
        assert rel_err(got, ref) < 2e-3
        cur = nxt


def test_chain_full_shape_two_tokens(orc):
    """8 chained full-shape layers (H 4096, I 2048, 256 experts top-8), 2 tokens, logits N(0,1).

    The chained scales (superblock scales 8x below the single-layer interval,
    shared expert std 0.01) keep each layer's output about 0.1, so the
    residual chain stays O(1)."""
    H = 4096
    shape = synth.Shape(H=H, I=2048, E=256, k=8)
    Ls, lays = [], []
    for l in range(LAYERS):
        L = synth.packed_layer(shape, 300 + l, router_std=1.0 / math.sqrt(H), device="cuda",
                               d_range=synth.CHAIN_D_RANGE, shared_std=synth.CHAIN_SHARED_STD)
        lay = m.MoELayer(H, 2048, 256, 8, 8)
        lay.load(L)
        Ls.append(L)
        lays.append(lay)
    x = synth.tokens(2, H, seed=11).cuda()
    inputs, out = _run_chain(lays, x)
    xo = x.cpu().numpy()
    for L, lay, xin in zip(Ls, lays, inputs):
        ids, _ = lay.route(xin)
        lg = orc.router_logits(xin.cpu().numpy(), L["W_r"].cpu().numpy())
        rid, _ = orc.topk_softmax(lg, 8)
        assert np.array_equal(ids.cpu().numpy(), rid)
    # independent oracle chain on the needed experts of each layer
    cur = xo.astype(np.float32)
    for L in Ls:
        lg = orc.router_logits(cur, L["W_r"].cpu().numpy())
        rid, _ = orc.topk_softmax(lg, 8)
        y, _, _ = orc.moe_forward(oracle_layer(L, experts=rid.ravel()), cur)
        cur = (cur.astype(np.float64) + y).astype(np.float32)
    assert rel_err(out.cpu().numpy(), cur) < 1e-4
