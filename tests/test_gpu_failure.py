"""Device-side failure paths, through the C ABI, with no GPU fault, trap or hang.

- A bounded wait that nothing satisfies gives up after its limit, records
  error bit 1 and the kernel returns: the host reads DS4MOE_ERR_TIMEOUT and
  the context keeps working.
- A grid with more magnitudes than the prefill plan's byte-permute selectors
  hold makes a prefill forward record error bit 2 and leave the output as it
  was; a later forward with a valid grid writes the output again.
"""
import ctypes

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


def _tiny(orc, max_tokens):
    L = synth.float_layer(synth.TINY, 0)
    L.update(pack_with_oracle(orc, L))
    lay = m.MoELayer(256, 128, 8, 2, max_tokens, act_dtype=m.DS4MOE_ACT_BF16)
    lay.load(L)
    return L, lay


def test_bounded_wait_times_out_and_context_survives(orc):
    L, lay = _tiny(orc, max_tokens=64)
    x = synth.tokens(4, 256, seed=3, dtype=torch.bfloat16).cuda()
    before = lay.forward(x).cpu()
    m.ds4moe_selftest_wait(lay.h)
    code = ctypes.c_int32(0)
    st = m.lib().ds4moe_get_device_error(lay.h, torch.cuda.current_stream().cuda_stream, ctypes.byref(code))
    assert st == -6 and code.value == 2             # DS4MOE_ERR_TIMEOUT, bit 1
    assert m.ds4moe_get_device_error(lay.h) == 0    # read and cleared
    after = lay.forward(x).cpu()                     # the context is still usable
    assert torch.equal(before, after)


def test_grid_with_five_magnitudes_refused_by_prefill(orc):
    L, lay = _tiny(orc, max_tokens=64)
    n = 40
    x = synth.tokens(n, 256, seed=4, dtype=torch.bfloat16).cuda()
    bad = L["grid"].clone()
    bad[0, :5] = torch.tensor([8, 25, 43, 60, 77], dtype=torch.uint8)   # five distinct magnitudes
    m.ds4moe_set_grid(lay.h, bad.cuda())
    out = torch.full((n, 256), float("nan"), device="cuda")
    m.ds4moe_forward(lay.h, x, out)
    torch.cuda.synchronize()
    assert torch.isnan(out).all()                    # left as it was
    # a valid grid again: the next forward writes out (before the error word is read)
    m.ds4moe_set_grid(lay.h, L["grid"].cuda())
    m.ds4moe_forward(lay.h, x, out)
    torch.cuda.synchronize()
    ref, _, _ = orc.moe_forward(oracle_layer(L), x.float().cpu().numpy(), mode=1)
    assert rel_err(out.cpu().numpy(), ref) < 2e-3
    code = m.ds4moe_get_device_error(lay.h)
    assert code & 4
