"""Routing through the no-allocation entry point (ds4moe_route_noalloc).

Callers that cannot allocate device memory -- a host that owns every device
buffer through its own pool, or code that must not stall the device with a
synchronizing allocation -- route with the library's static device scratch.
This checks that entry point against ds4moe_route on two calls in a row with
different tokens (the second call must not see the first call's scratch),
through the C ABI, and that it needs no bound workspace.  It lives in its own
file, collected last, and passes on its own in a fresh process as well as
after the others.
"""
import numpy as np
import pytest
import torch

import bit_quantized_moe_softmax_b200 as m
from bit_quantized_moe_softmax_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_moe_softmax_b200 import build

    build.build()


def _layer(E, k, H=256, I=128, max_tokens=8):
    L = synth.float_layer(synth.Shape(H=H, I=I, E=E, k=k), seed=3)
    lay = m.MoELayer(H, I, E, k, max_tokens)
    lay.load(L)
    return lay


@pytest.mark.parametrize("E,k,n", [(8, 2, 4), (256, 8, 8)])
def test_route_noalloc_matches_route_twice(E, k, n):
    lay = _layer(E, k, H=4096 if E == 256 else 256)
    for call, seed in enumerate((11, 12)):
        x = synth.tokens(n, lay.H, seed=seed).cuda()
        ids_ref, w_ref = lay.route(x)
        ids = torch.full((n, k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((n, k), -1.0, dtype=torch.float32, device="cuda")
        m.ds4moe_route_noalloc(lay.h, x, ids, w)
        torch.cuda.synchronize()
        assert np.array_equal(ids.cpu().numpy(), ids_ref.cpu().numpy()), call
        assert np.abs(w.cpu().numpy() - w_ref.cpu().numpy()).max() <= 1e-6, call
    assert m.ds4moe_get_device_error(lay.h) == 0


def test_route_noalloc_without_workspace():
    """A handle bound to its weight buffer alone (no workspace) routes through
    the static scratch; calls that need the workspace are refused."""
    E, k, H, n = 8, 2, 256, 3
    L = synth.float_layer(synth.Shape(H=H, I=128, E=E, k=k), seed=4)
    ref = _layer(E, k)
    ref.load(L)
    h = m.ds4moe_create(H, 128, E, k, 8)
    try:
        wbuf = torch.empty(m.ds4moe_weight_bytes(h), dtype=torch.uint8, device="cuda")
        m.ds4moe_bind(h, wbuf, None)
        m.ds4moe_set_grid(h, L["grid"].cuda())
        m.ds4moe_set_router(h, L["W_r"].cuda())
        x = synth.tokens(n, H, seed=5).cuda()
        ids = torch.empty(n, k, dtype=torch.int32, device="cuda")
        w = torch.empty(n, k, dtype=torch.float32, device="cuda")
        m.ds4moe_route_noalloc(h, x, ids, w)
        ids_ref, w_ref = ref.route(x)
        torch.cuda.synchronize()
        assert torch.equal(ids.cpu(), ids_ref.cpu())
        assert np.abs(w.cpu().numpy() - w_ref.cpu().numpy()).max() <= 1e-6
        assert m.ds4moe_get_device_error(h) == 0
        with pytest.raises(m.Ds4MoeError) as ei:
            m.ds4moe_route(h, x, ids, w)
        assert ei.value.status == -4 and "workspace not bound" in str(ei.value)
    finally:
        m.ds4moe_destroy(h)


def test_route_noalloc_rejects_more_tokens_than_decode_max():
    # n_tokens * n_experts <= 8192 always holds for a valid handle (at most 8
    # decode tokens times at most 1024 experts), so the limit a caller meets is
    # decode_max; 8 tokens of 1024 experts fill the scratch exactly.
    lay = _layer(E=1024, k=2, H=256, I=128, max_tokens=16)
    x = synth.tokens(8, 256, seed=1).cuda()
    ids = torch.empty(8, 2, dtype=torch.int32, device="cuda")
    w = torch.empty(8, 2, dtype=torch.float32, device="cuda")
    m.ds4moe_route_noalloc(lay.h, x, ids, w)          # 8 * 1024 = 8192: at the limit
    with pytest.raises(m.Ds4MoeError) as ei:          # more tokens than the decode plan
        m.ds4moe_route_noalloc(lay.h, synth.tokens(9, 256, seed=2).cuda(),
                               torch.empty(9, 2, dtype=torch.int32, device="cuda"),
                               torch.empty(9, 2, device="cuda"))
    assert ei.value.status == -1 and "decode_max" in str(ei.value)
