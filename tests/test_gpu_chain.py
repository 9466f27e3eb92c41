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


# ------------------------------------------------------------------ one call for the whole chain
def _chain_call(lays, x, n):
    out = torch.empty(n, lays[0].H, device="cuda")
    work = torch.empty(2, n, lays[0].H, device="cuda")
    m.ds4moe_forward_chain([lay.h for lay in lays], x, out, work)
    torch.cuda.synchronize()
    for lay in lays:
        assert m.ds4moe_get_device_error(lay.h) == 0
    return out


@pytest.mark.parametrize("n", [1, 2, 8])
def test_forward_chain_equals_layer_by_layer(orc, n):
    """ds4moe_forward_chain (layers launched as programmatic dependents of one another, each prologue
    waiting on the previous combine's count) gives the layer-by-layer residual chain bit for bit,
    and so the oracle's chain within 1e-4; repeated calls reuse the counters."""
    Ls, lays = _tiny_chain(orc)
    x = synth.tokens(n, 256, seed=40 + n).cuda()
    _, seq = _run_chain(lays, x)
    for _ in range(3):
        out = _chain_call(lays, x, n)
        assert torch.equal(out, seq)
    ref, _, _ = orc.chain_forward([oracle_layer(L) for L in Ls], x.cpu().numpy())
    assert rel_err(out.cpu().numpy(), ref) < 1e-4


def test_forward_chain_mixed_bits_and_steering(orc):
    """A chain whose layers alternate 2-bit and 4-bit experts, one layer steered (its combine is the
    one-CTA-per-token kernel, which the next layer counts), a bf16 first layer."""
    from tests._util import pack_q4_with_oracle

    H = 256
    lays, Ls = [], []
    for l in range(4):
        L = synth.float_layer(synth.Shape(H=H, I=256, E=8, k=2), 500 + l, router_std=1.0 / math.sqrt(H))
        bits = 4 if l % 2 else 0
        L.update(pack_q4_with_oracle(orc, L) if bits == 4 else pack_with_oracle(orc, L))
        lay = m.MoELayer(H, 256, 8, 2, 8, act_dtype=m.DS4MOE_ACT_BF16 if l == 0 else m.DS4MOE_ACT_F32,
                         expert_bits=bits)
        lay.load(L if bits != 4 else {**L, "grid": None})
        lays.append(lay)
        Ls.append(L)
    v = synth.normal((H,), 1.0, synth.gen(7))
    lays[2].set_steering((v / v.double().norm().float()).cuda().contiguous(), 0.5)
    x = synth.tokens(3, H, seed=8, dtype=torch.bfloat16).cuda()
    cur = x
    for lay in lays:
        cur = lay.forward(cur, residual=True)
    out = _chain_call(lays, x, 3)
    assert torch.equal(out, cur)


def test_forward_chain_full_shape_two_tokens():
    """8 full-shape layers, 2 tokens: the one-call chain equals the layer-by-layer chain bit for bit."""
    H = 4096
    shape = synth.Shape(H=H, I=2048, E=256, k=8)
    lays = []
    for l in range(LAYERS):
        L = synth.packed_layer(shape, 300 + l, router_std=1.0 / math.sqrt(H), device="cuda",
                               d_range=synth.CHAIN_D_RANGE, shared_std=synth.CHAIN_SHARED_STD)
        lay = m.MoELayer(H, 2048, 256, 8, 8)
        lay.load(L)
        lays.append(lay)
        del L
    x = synth.tokens(2, H, seed=11).cuda()
    _, seq = _run_chain(lays, x)
    for _ in range(2):
        assert torch.equal(_chain_call(lays, x, 2), seq)


def test_forward_chain_argument_errors(orc):
    Ls, lays = _tiny_chain(orc)
    x = synth.tokens(2, 256, seed=1).cuda()
    out = torch.empty(2, 256, device="cuda")
    work = torch.empty(2, 2, 256, device="cuda")
    with pytest.raises(m.Ds4MoeError) as ei:   # one handle twice
        m.ds4moe_forward_chain([lays[0].h, lays[0].h], x, out, work)
    assert ei.value.status == -1
    with pytest.raises(m.Ds4MoeError) as ei:   # work overlaps out
        m.ds4moe_forward_chain([lay.h for lay in lays], x, work[0], work)
    assert ei.value.status == -1
    bf = m.MoELayer(256, 128, 8, 2, 8, act_dtype=m.DS4MOE_ACT_BF16)
    bf.load(Ls[1])
    with pytest.raises(m.Ds4MoeError) as ei:   # a bf16 layer after the first
        m.ds4moe_forward_chain([lays[0].h, bf.h], x, out, work)
    assert ei.value.status == -3
