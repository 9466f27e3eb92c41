"""GPU parity of the decode (fp32 GEMV) plan against the CPU oracle, through the C ABI.

Bars: packed bytes, dequantized weights and routed expert ids bit-exact;
router weights within 1e-6; layer outputs within 1e-4 of max|ref|
(rel = max|gpu - ref| / max|ref|).
"""
import numpy as np
import pytest
import torch

import bit_quantized_moe_softmax_b200 as m
from bit_quantized_moe_softmax_b200 import synth
from tests._util import oracle_layer, pack_with_oracle, rel_err

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_moe_softmax_b200 import build

    build.build()


def _tiny(orc, E=8, k=2, seed=0, bias=False, shared=True, router_std=0.02):
    shape = synth.Shape(H=256, I=128, E=E, k=k, shared=shared)
    b = synth.zipf_bias(E, 1.1, seed) if bias else None
    L = synth.float_layer(shape, seed, router_std=router_std, bias=b)
    L.update(pack_with_oracle(orc, L))
    return L


def _layer_on_gpu(L, max_tokens=8, act=m.DS4MOE_ACT_F32, decode_max=0):
    lay = m.MoELayer(L["H"], L["I"], L["E"], L["k"], max_tokens, act_dtype=act,
                     has_shared=L.get("sh_gate") is not None, has_bias=L.get("b_r") is not None,
                     decode_max=decode_max)
    lay.load(L)
    return lay


# ------------------------------------------------------------------ packers
@pytest.mark.parametrize("nblocks", [1, 3, 128, 1000])
def test_pack_q2k_bytes_match_oracle(orc, nblocks):
    g = synth.gen(nblocks)
    w = synth.normal((nblocks * 256,), 0.02, g)
    w[:256] *= 0                      # an all-zero block
    w[256:272] = torch.abs(w[256:272])  # a sub-block with no negatives
    ref = orc.pack_q2k(w.numpy())
    out = torch.empty(nblocks, 84, dtype=torch.uint8, device="cuda")
    m.ds4moe_pack_q2k(w.cuda(), out)
    assert np.array_equal(out.cpu().numpy(), ref)


@pytest.mark.parametrize("nblocks", [1, 3, 128, 517])
def test_pack_iq2_bytes_match_oracle(orc, nblocks):
    g = synth.gen(100 + nblocks)
    w = synth.normal((nblocks * 256,), 0.02, g)
    w[:256] *= 0
    if nblocks > 1:
        w[300] = -0.0
    grid = synth.grid_table(0)
    ref = orc.pack_iq2xxs(w.numpy(), grid.numpy())
    out = torch.empty(nblocks, 66, dtype=torch.uint8, device="cuda")
    m.ds4moe_pack_iq2xxs(w.cuda(), grid.cuda(), out)
    assert np.array_equal(out.cpu().numpy(), ref)


# ------------------------------------------------------------------ dequant hook
@pytest.mark.parametrize("as_bf16", [0, 1])
def test_dequant_bit_exact_tiny(orc, as_bf16):
    L = _tiny(orc)
    lay = _layer_on_gpu(L)
    grid = L["grid"].numpy()
    for e in (0, 5):
        for which, ref in ((0, orc.dequant_iq2xxs(L["gate"][e].numpy(), grid).reshape(128, 256)),
                           (1, orc.dequant_iq2xxs(L["up"][e].numpy(), grid).reshape(128, 256)),
                           (2, orc.dequant_q2k(L["down"][e].numpy()).reshape(256, 128))):
            got = lay.dequant(e, which, bool(as_bf16)).float().cpu().numpy()
            exp = orc.bf16_round(ref) if as_bf16 else ref
            assert np.array_equal(got, exp), (e, which)


def test_dequant_bit_exact_full_shape(orc):
    shape = synth.Shape(H=4096, I=2048, E=2, k=1, shared=False)
    L = synth.packed_layer(shape, 1, device="cuda")
    lay = _layer_on_gpu(L, max_tokens=1)
    grid = L["grid"].numpy()
    e = 1
    ref_g = orc.dequant_iq2xxs(L["gate"][e].cpu().numpy(), grid).reshape(2048, 4096)
    assert np.array_equal(lay.dequant(e, 0).cpu().numpy(), ref_g)
    ref_d = orc.dequant_q2k(L["down"][e].cpu().numpy()).reshape(4096, 2048)
    assert np.array_equal(lay.dequant(e, 2).cpu().numpy(), ref_d)
    assert np.array_equal(lay.dequant(e, 2, True).float().cpu().numpy(), orc.bf16_round(ref_d))


# ------------------------------------------------------------------ routing
@pytest.mark.parametrize("n,bias", [(1, False), (4, False), (8, True)])
def test_route_ids_exact(orc, n, bias):
    L = _tiny(orc, bias=bias)
    lay = _layer_on_gpu(L)
    x = synth.tokens(n, 256, seed=n)
    ids, w = lay.route(x.cuda())
    lg = orc.router_logits(x.numpy(), L["W_r"].numpy(), None if not bias else L["b_r"].numpy())
    rid, rw = orc.topk_softmax(lg, L["k"])
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.abs(w.cpu().numpy() - rw).max() < 1e-6


def test_route_full_shape_logits_order(orc):
    shape = synth.Shape(H=4096, I=256, E=256, k=8, shared=False)
    L = synth.packed_layer(shape, 2, device="cuda")
    lay = _layer_on_gpu(L, max_tokens=8)
    x = synth.tokens(8, 4096, seed=3)
    ids, w = lay.route(x.cuda())
    lg = orc.router_logits(x.numpy(), L["W_r"].cpu().numpy())
    rid, rw = orc.topk_softmax(lg, 8)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.abs(w.cpu().numpy() - rw).max() < 1e-6


# ------------------------------------------------------------------ forward
@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_forward_tiny_matches_oracle(orc, n):
    L = _tiny(orc)
    lay = _layer_on_gpu(L)
    x = synth.tokens(n, 256, seed=10 + n)
    out = lay.forward(x.cuda()).cpu().numpy()
    ref, _, _ = orc.moe_forward(oracle_layer(L), x.numpy())
    assert rel_err(out, ref) < TOL


# n = 1 takes the one-token producer (shared-expert and routed gate/up tasks from two queues, in turn),
# n = 3 the single-queue one
@pytest.mark.parametrize("n", [1, 3])
@pytest.mark.parametrize("variant", ["bias", "no_shared", "one_expert", "k_equals_E", "bf16_act", "unit_logits"])
def test_forward_tiny_variants(orc, variant, n):
    kw = dict(bias=variant == "bias", shared=variant != "no_shared")
    if variant == "one_expert":
        kw.update(E=1, k=1)
    if variant == "k_equals_E":
        kw.update(E=4, k=4)
    if variant == "unit_logits":
        kw.update(router_std=1 / 16)
    L = _tiny(orc, **kw)
    act = m.DS4MOE_ACT_BF16 if variant == "bf16_act" else m.DS4MOE_ACT_F32
    lay = _layer_on_gpu(L, act=act)
    x = synth.tokens(n, 256, seed=21, dtype=torch.bfloat16 if act else torch.float32)
    out = lay.forward(x.cuda()).cpu().numpy()
    ref, _, _ = orc.moe_forward(oracle_layer(L), x.float().numpy())
    assert rel_err(out, ref) < TOL


def test_forward_all_tokens_one_expert(orc):
    # every token chooses experts 3 and 6: one expert read serves all tokens
    L = _tiny(orc)
    L["W_r"] = torch.zeros_like(L["W_r"])
    L["b_r"] = torch.tensor([0, 0, 0, 2.0, 0, 0, 1.0, 0])
    lay = _layer_on_gpu(L)
    x = synth.tokens(8, 256, seed=5)
    out = lay.forward(x.cuda()).cpu().numpy()
    ref, ids, _ = orc.moe_forward(oracle_layer(L), x.numpy())
    assert np.all(ids == [3, 6])
    assert rel_err(out, ref) < TOL


def test_forward_repeatable_and_deterministic(orc):
    L = _tiny(orc)
    lay = _layer_on_gpu(L)
    x = synth.tokens(4, 256, seed=7).cuda()
    outs = [lay.forward(x).cpu().numpy() for _ in range(4)]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_forward_host_buffers(orc):
    L = _tiny(orc)
    lay = _layer_on_gpu(L)
    x = synth.tokens(4, 256, seed=8).pin_memory()
    out = torch.empty(4, 256, dtype=torch.float32).pin_memory()
    m.ds4moe_forward_host(lay.h, x, out)
    ref = lay.forward(x.cuda()).cpu()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("n,max_tokens", [(3, 8), (40, 64)])
def test_forward_host_async_pipeline(orc, n, max_tokens):
    """Pipelined host-buffer calls: six calls in flight over the two staging
    slots (decode and prefill plans), a blocking call in between; every
    result equals the device-buffer forward of the same input bit for bit."""
    L = _tiny(orc)
    lay = _layer_on_gpu(L, max_tokens=max_tokens)
    xs = [synth.tokens(n, 256, seed=100 + i).pin_memory() for i in range(6)]
    outs = [torch.full((n, 256), float("nan"), dtype=torch.float32).pin_memory() for _ in range(6)]
    for i in range(3):
        m.ds4moe_forward_host_async(lay.h, xs[i], outs[i])
    m.ds4moe_forward_host(lay.h, xs[3], outs[3])
    for i in range(4, 6):
        m.ds4moe_forward_host_async(lay.h, xs[i], outs[i])
    m.ds4moe_host_sync(lay.h)
    for i in range(6):
        assert torch.equal(outs[i], lay.forward(xs[i].cuda()).cpu()), i
    m.ds4moe_host_sync(lay.h)   # nothing pending: returns at once


@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_forward_full_decode_shape(orc, n):
    """n tokens through a full-size layer (H 4096, I 2048, 256 experts top-8, bf16 shared), in the
    launch configuration the bench times: n = 1 is the decode step, 2 / 4 / 8 the MTP-verify sizes
    (8 tokens: about 57 distinct experts, some chosen by two tokens)."""
    L = synth.packed_layer(synth.FULL, 0, device="cuda")
    lay = _layer_on_gpu(L, max_tokens=8)
    x = synth.tokens(n, 4096, seed=1 + n)
    out = lay.forward(x.cuda()).cpu().numpy()
    ids_gpu, _ = lay.route(x.cuda())
    lg = orc.router_logits(x.numpy(), L["W_r"].cpu().numpy())
    rid, _ = orc.topk_softmax(lg, 8)
    assert np.array_equal(ids_gpu.cpu().numpy(), rid)
    ref, ids, _ = orc.moe_forward(oracle_layer(L, experts=rid.ravel()), x.numpy())
    assert np.array_equal(ids, rid)
    assert rel_err(out, ref) < TOL


def test_forward_full_shape_expert_of_every_token(orc):
    """Eight tokens that all choose expert 17 (router bias): one expert serves more tokens than one
    routed entry holds, so its weights are read by several entries; bf16 activations."""
    bias = torch.zeros(256)
    bias[17] = 30.0
    L = synth.packed_layer(synth.FULL, 4, bias=bias, device="cuda")
    lay = _layer_on_gpu(L, max_tokens=8, act=m.DS4MOE_ACT_BF16)
    x = synth.tokens(8, 4096, seed=9, dtype=torch.bfloat16)
    out = lay.forward(x.cuda()).cpu().numpy()
    lg = orc.router_logits(x.float().numpy(), L["W_r"].cpu().numpy(), bias.numpy())
    rid, _ = orc.topk_softmax(lg, 8)
    assert np.all(rid[:, 0] == 17)
    ref, ids, _ = orc.moe_forward(oracle_layer(L, experts=rid.ravel()), x.float().numpy())
    assert rel_err(out, ref) < TOL


# ------------------------------------------------------------------ host-side checks
def test_argument_errors(orc):
    L = _tiny(orc)
    lay = _layer_on_gpu(L, max_tokens=4)
    x = synth.tokens(5, 256, seed=1).cuda()
    out = torch.empty(5, 256, device="cuda")
    with pytest.raises(m.Ds4MoeError) as ei:
        m.ds4moe_forward(lay.h, x, out)
    assert ei.value.status == -1
    xb = torch.empty(4 * 256 + 1, device="cuda")[1:].view(4, 256)
    with pytest.raises(m.Ds4MoeError) as ei:
        m.ds4moe_forward(lay.h, xb, out[:4])
    assert ei.value.status == -2
    m.ds4moe_forward(lay.h, x[:0], out[:0])   # n = 0 is a no-op
    fresh = m.MoELayer(256, 128, 8, 2, 4)
    with pytest.raises(m.Ds4MoeError) as ei:
        fresh.forward(x[:2])
    assert ei.value.status == -4
    assert m.ds4moe_get_device_error(lay.h) == 0
