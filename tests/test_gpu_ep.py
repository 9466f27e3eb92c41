"""GPU halves of expert parallelism on one device, against the one-GPU layer and the oracle.

ds4moe_forward_routed (the layer with the caller's routing) is checked
against the oracle's experts: out[t] = shared(x_t) + sum_j w[t][j]
expert_{ids[t][j]}(x_t), each expert output and the shared output taken from
oracle layers of one expert.  Then a layer's experts are split over two
shards (two handles over contiguous expert ranges, as two ranks would hold
them); the rows of each shard go through its handle, come back in slot order
and are summed by ds4moe_combine_slots onto the shared expert's output: on
the decode plan the result equals the one-GPU layer bit for bit (the same
kernels on the same rows, the same combine order).  The exchange itself is
covered by the gloo tests.  Bars: decode 1e-4, tensor-core plan 2e-3 of
max|ref|.
"""
import numpy as np
import pytest
import torch

import bit_quantized_moe_softmax_b200 as m
from bit_quantized_moe_softmax_b200 import ep, synth
from tests._util import oracle_layer, pack_with_oracle, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_moe_softmax_b200 import build

    build.build()


def _tiny(orc, seed=0):
    L = synth.float_layer(synth.Shape(H=256, I=128, E=8, k=2), seed)
    L.update(pack_with_oracle(orc, L))
    return L


def _full_layer(L, max_tokens):
    lay = m.MoELayer(L["H"], L["I"], L["E"], L["k"], max_tokens)
    lay.load(L)
    return lay


def _oracle_routed(orc, L, x, ids, w):
    """shared(x_t) + sum_j w[t][j] expert_{ids[t][j]}(x_t) from oracle layers of one expert."""
    base = oracle_layer(L)
    n, k = ids.shape
    out = np.zeros((n, L["H"]))
    for t in range(n):
        xt = x[t:t + 1]
        for j in range(k):
            e = int(ids[t, j])
            one = dict(base, E=1, k=1, W_r=np.zeros((1, L["H"]), np.float32), b_r=None, gate=[base["gate"][e]],
                       up=[base["up"][e]], down=[base["down"][e]], sh_gate=None, sh_up=None, sh_down=None)
            y, _, _ = orc.moe_forward(one, xt)
            out[t] += w[t, j] * y[0]
        sh = dict(base, E=1, k=1, W_r=np.zeros((1, L["H"]), np.float32), b_r=None, gate=[base["gate"][0]],
                  up=[base["up"][0]], down=[base["down"][0]])
        y_sh_plus, _, _ = orc.moe_forward(sh, xt)
        one0 = dict(sh, sh_gate=None, sh_up=None, sh_down=None)
        y0, _, _ = orc.moe_forward(one0, xt)
        out[t] += y_sh_plus[0] - y0[0]
    return out


@pytest.mark.parametrize("n", [1, 3, 8])
def test_forward_routed_matches_oracle(orc, n):
    L = _tiny(orc)
    lay = _full_layer(L, 8)
    g = synth.gen(60 + n)
    ids = torch.randint(0, 8, (n, 2), generator=g, dtype=torch.int32)
    ids[0, 1] = ids[0, 0]                      # an expert twice in one token
    w = torch.rand(n, 2, generator=g)
    x = synth.tokens(n, 256, seed=61 + n)
    out = torch.empty(n, 256, device="cuda")
    m.ds4moe_forward_routed(lay.h, x.cuda(), ids.cuda(), w.cuda(), out)
    torch.cuda.synchronize()
    assert m.ds4moe_get_device_error(lay.h) == 0
    ref = _oracle_routed(orc, L, x.numpy(), ids.numpy(), w.numpy())
    assert rel_err(out.cpu().numpy(), ref) < 1e-4


def test_forward_routed_router_ids_equal_forward(orc):
    """Given the router's own ids and weights, the routed forward is the forward, bit for bit."""
    L = _tiny(orc, seed=3)
    for n, cap in ((4, 8), (40, 64)):
        lay = _full_layer(L, cap)
        x = synth.tokens(n, 256, seed=70 + n).cuda()
        ids, w = lay.route(x)
        out = torch.empty(n, 256, device="cuda")
        m.ds4moe_forward_routed(lay.h, x, ids, w, out)
        assert torch.equal(out, lay.forward(x)), n


def test_forward_routed_bad_id_is_flagged(orc):
    L = _tiny(orc)
    lay = _full_layer(L, 8)
    x = synth.tokens(2, 256, seed=5).cuda()
    ids = torch.tensor([[1, 9], [2, 3]], dtype=torch.int32, device="cuda")
    w = torch.tensor([[0.5, 0.5], [0.5, 0.5]], device="cuda")
    out = torch.empty(2, 256, device="cuda")
    m.ds4moe_forward_routed(lay.h, x, ids, w, out)
    assert m.ds4moe_get_device_error(lay.h) == 1   # bit 0: an index check failed (read and cleared)
    assert m.ds4moe_get_device_error(lay.h) == 0
    # the bad slot counts as expert 0 with weight 0: token 0 is shared + 0.5 expert 1
    ids2 = torch.tensor([[1, 0], [2, 3]], dtype=torch.int32, device="cuda")
    w2 = torch.tensor([[0.5, 0.0], [0.5, 0.5]], device="cuda")
    out2 = torch.empty(2, 256, device="cuda")
    m.ds4moe_forward_routed(lay.h, x, ids2, w2, out2)
    assert torch.equal(out, out2)


def _split_layer_forward(L, x, ids, w, shards, max_rows):
    """The layer on two expert shards: rows to their shard, back in slot order, combined on the device."""
    n, k = ids.shape
    H = L["H"]
    slots_e = ids.reshape(-1).long()
    ys = torch.empty(n * k, H, device="cuda")
    for sh in shards:
        sel = torch.nonzero((slots_e >= sh.first) & (slots_e < sh.first + sh.count)).reshape(-1)
        if sel.numel():
            ys[sel] = sh(x[sel // k].contiguous(), slots_e[sel])
    # the shared expert's output: a handle with the shared expert and one routed expert of weight 0
    shl = m.MoELayer(H, L["I"], 1, 1, max(8, n))
    shl.load(dict(L, E=1, k=1, W_r=L["W_r"][:1], b_r=None, gate=L["gate"][:1], up=L["up"][:1], down=L["down"][:1]))
    base = torch.empty(n, H, device="cuda")
    m.ds4moe_forward_routed(shl.h, x, torch.zeros(n, 1, dtype=torch.int32, device="cuda"),
                            torch.zeros(n, 1, device="cuda"), base)
    out = torch.empty(n, H, device="cuda")
    m.ds4moe_combine_slots(ys, w.contiguous(), base, out)
    return out


@pytest.mark.parametrize("n", [1, 3])
def test_two_shards_equal_one_gpu_layer_decode(orc, n):
    L = _tiny(orc, seed=9)
    lay = _full_layer(L, 8)
    x = synth.tokens(n, 256, seed=90 + n).cuda()
    ids, w = lay.route(x)
    shards = [ep.GpuExpertShard(L, 8, r, 2, max_rows=8) for r in range(2)]
    out = _split_layer_forward(L, x, ids, w, shards, 8)
    assert torch.equal(out, lay.forward(x))


def test_two_shards_tensor_core_plan(orc):
    """64 tokens (128 slots): each shard's rows go through the tensor-core plan in one call."""
    L = _tiny(orc, seed=11)
    lay = _full_layer(L, 64)
    x = synth.tokens(64, 256, seed=12).cuda()
    ids, w = lay.route(x)
    shards = [ep.GpuExpertShard(L, 8, r, 2, max_rows=128) for r in range(2)]
    out = _split_layer_forward(L, x, ids, w, shards, 128)
    ref = lay.forward(x)
    assert rel_err(out.cpu().numpy(), ref.cpu().numpy()) < 2e-3


def test_combine_slots_order_and_alias():
    """combine_slots adds the slots in order with one FMA each; out may alias base."""
    g = synth.gen(3)
    n, k, H = 5, 3, 64
    y = torch.randn(n * k, H, generator=g).cuda()
    w = torch.rand(n, k, generator=g).cuda()
    base = torch.randn(n, H, generator=g).cuda()
    out = torch.empty(n, H, device="cuda")
    m.ds4moe_combine_slots(y, w, base, out)
    ref = base.clone()
    for j in range(k):   # torch.addcmul rounds the product first; the kernel fuses: compare at 1e-6
        ref = ref + w[:, j:j + 1] * y.view(n, k, H)[:, j]
    assert torch.allclose(out, ref, rtol=1e-6, atol=1e-6)
    b2 = base.clone()
    m.ds4moe_combine_slots(y, w, b2, b2)
    assert torch.equal(b2, out)
    z = torch.empty(n, H, device="cuda")
    m.ds4moe_combine_slots(y, w, None, z)
    assert torch.allclose(z + base, out, rtol=1e-5, atol=1e-5)
