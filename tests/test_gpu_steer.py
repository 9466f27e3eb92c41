"""GPU parity of directional steering of the layer output (y -= F v (v . y)) against the CPU oracle.

The pages' server applies it after FFN outputs with one binary32 direction
vector per layer; here it is fused into the combine kernel of both plans.
Bars: decode plan 1e-4 of max|ref|, prefill plan 2e-3 (bf16 reading).
"""
import numpy as np
import pytest
import torch

import bit_quantized_moe_softmax_b200 as m
from bit_quantized_moe_softmax_b200 import synth
from tests._util import oracle_layer, pack_with_oracle, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_moe_softmax_b200 import build

    build.build()


def _tiny(orc, max_tokens=8, act=m.DS4MOE_ACT_F32):
    L = synth.float_layer(synth.Shape(H=256, I=128, E=8, k=2), 4)
    L.update(pack_with_oracle(orc, L))
    lay = m.MoELayer(256, 128, 8, 2, max_tokens, act_dtype=act)
    lay.load(L)
    return L, lay


def _direction(seed=1):
    return synth.normal((256,), 1.0 / 16, synth.gen(seed), "cpu")   # |v| about 1


@pytest.mark.parametrize("n,F", [(1, 1.0), (4, 0.6), (8, 2.0)])
def test_steer_decode(orc, n, F):
    L, lay = _tiny(orc)
    v = _direction()
    lay.set_steering(v.cuda(), F)
    x = synth.tokens(n, 256, seed=30 + n)
    out = lay.forward(x.cuda()).cpu().numpy()
    y, _, _ = orc.moe_forward(oracle_layer(L), x.numpy())
    ref = orc.steer(y, v.numpy(), F)
    assert rel_err(out, ref) < 1e-4
    # with F = 1 and a unit direction the output has no component along v
    if F == 1.0:
        vn = v.double().numpy() / np.linalg.norm(v.double().numpy())
        lay.set_steering(torch.from_numpy(vn.astype(np.float32)).cuda(), 1.0)
        o1 = lay.forward(x.cuda()).double().cpu().numpy()
        assert np.abs(o1 @ vn).max() < 1e-5 * np.abs(o1).max() * 16


def test_steer_prefill(orc):
    L, lay = _tiny(orc, max_tokens=64)
    v = _direction(2)
    lay.set_steering(v.cuda(), 0.8)
    x = synth.tokens(64, 256, seed=5)
    out = lay.forward(x.cuda()).cpu().numpy()
    y, _, _ = orc.moe_forward(oracle_layer(L), x.numpy(), mode=1)
    assert rel_err(out, orc.steer(y, v.numpy(), 0.8)) < 2e-3


def test_steer_with_residual_and_off_switch(orc):
    L, lay = _tiny(orc)
    x = synth.tokens(4, 256, seed=6).cuda()
    plain = lay.forward(x)
    v = _direction(3)
    lay.set_steering(v.cuda(), 0.5)
    st = lay.forward(x)
    r = lay.forward(x, residual=True)
    assert torch.equal(r, x + st)
    assert torch.equal(lay.forward(x), st)          # fixed summation order: repeats bitwise
    lay.set_steering(None)
    assert torch.equal(lay.forward(x), plain)       # off again: the plain combine
    lay.set_steering(v.cuda(), 0.0)
    assert torch.equal(lay.forward(x), plain)


def test_steer_plan_names_and_errors(orc):
    L, lay = _tiny(orc, max_tokens=64)
    v = _direction(4).cuda()
    lay.set_steering(v, 1.0)
    assert m.ds4moe_plan_kernel(lay.h, 1, m.ds4moe_plan_launches(lay.h, 1) - 1) == "k_combine_steer_decode"
    assert m.ds4moe_plan_kernel(lay.h, 64, m.ds4moe_plan_launches(lay.h, 64) - 1) == "k_combine_steer_prefill"
    with pytest.raises(m.Ds4MoeError):
        m.ds4moe_set_steering(lay.h, v, float("inf"))
