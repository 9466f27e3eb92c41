"""GPU parity of the 4-bit routed-expert variant (Q4_K-style gate, up and down
blocks; decode plan) against the CPU oracle, through the C ABI.

Bars: packed bytes bit-exact; dequantized weights bit-exact (binary32, and
bf16 of them); each weight the projection kernel multiplies bit-exact (one-hot
probes: one code times 1.0 minus one min term, a single rounding on both
sides); layer outputs within 1e-4 of max|ref| (rel = max|gpu - ref| /
max|ref|), the decode plan's bar.
"""
import numpy as np
import pytest
import torch

import bit_quantized_moe_softmax_b200 as m
from bit_quantized_moe_softmax_b200 import synth
from tests._util import oracle_layer, pack_q4_with_oracle, rel_err

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_moe_softmax_b200 import build

    build.build()


def _tiny(orc, E=8, k=2, seed=0, bias=False, shared=True, H=256, I=256):
    shape = synth.Shape(H=H, I=I, E=E, k=k, shared=shared)
    b = synth.zipf_bias(E, 1.1, seed) if bias else None
    L = synth.float_layer(shape, seed, bias=b)
    L.update(pack_q4_with_oracle(orc, L))
    return L


def _load(L, max_tokens=8, act=m.DS4MOE_ACT_F32):
    lay = m.MoELayer(L["H"], L["I"], L["E"], L["k"], max_tokens, act_dtype=act,
                     has_shared=L.get("sh_gate") is not None, has_bias=L.get("b_r") is not None,
                     expert_bits=4)
    lay.load({**L, "grid": None})   # 4-bit layers need no grid
    return lay


# ------------------------------------------------------------------ packer
@pytest.mark.parametrize("nblocks", [1, 3, 128, 517])
def test_pack_q4k_bytes_match_oracle(orc, nblocks):
    g = synth.gen(200 + nblocks)
    w = synth.normal((nblocks * 256,), 0.02, g)
    w[:256] *= 0                        # an all-zero block
    w[256:288] = torch.abs(w[256:288])  # a sub-block with no negatives (lo = 0)
    if nblocks > 2:
        w[544:576] = -torch.abs(w[544:576])   # one with no positives (hi = 0)
    ref = orc.pack_q4k(w.numpy())
    out = torch.empty(nblocks, 144, dtype=torch.uint8, device="cuda")
    m.ds4moe_pack_q4k(w.cuda(), out)
    assert np.array_equal(out.cpu().numpy(), ref)


def test_pack_q4k_argument_errors():
    w = torch.zeros(300, device="cuda")
    out = torch.empty(2, 144, dtype=torch.uint8, device="cuda")
    with pytest.raises(m.Ds4MoeError) as ei:
        m.ds4moe_pack_q4k(w, out)
    assert ei.value.status == -1


# ------------------------------------------------------------------ dequant hook
@pytest.mark.parametrize("as_bf16", [0, 1])
def test_dequant_q4_bit_exact_tiny(orc, as_bf16):
    L = _tiny(orc)
    lay = _load(L)
    for e in (0, 5):
        for which, name, shp in ((0, "gate", (256, 256)), (1, "up", (256, 256)), (2, "down", (256, 256))):
            ref = orc.dequant_q4k(L[name][e].numpy()).reshape(shp)
            got = lay.dequant(e, which, bool(as_bf16)).float().cpu().numpy()
            assert np.array_equal(got, orc.bf16_round(ref) if as_bf16 else ref), (e, which)


def test_dequant_q4_bit_exact_full_shape(orc):
    shape = synth.Shape(H=4096, I=2048, E=2, k=1, shared=False)
    L = synth.packed_layer(shape, 1, device="cuda", expert_bits=4)
    lay = _load(L, max_tokens=1)
    e = 1
    assert np.array_equal(lay.dequant(e, 1).cpu().numpy(),
                          orc.dequant_q4k(L["up"][e].cpu().numpy()).reshape(2048, 4096))
    assert np.array_equal(lay.dequant(e, 2).cpu().numpy(),
                          orc.dequant_q4k(L["down"][e].cpu().numpy()).reshape(4096, 2048))


# ------------------------------------------------------------------ weights the kernel multiplies
def _edge_blocks(nb: int, seed: int) -> torch.Tensor:
    """Random blocks with hand-set edges: zero d, zero dmin, negative and
    subnormal scales, all codes 15 with the largest fields (63), all codes 0."""
    b = synth.random_q4k_blocks(nb, synth.gen(seed))
    half = lambda v: torch.tensor([v], dtype=torch.float16).view(torch.uint8)
    b[0, 0:2] = half(0.0)
    b[1, 2:4] = half(0.0)
    b[2, 0:2] = half(-3e-4)
    b[3, 0:2] = half(2.0 ** -20)       # subnormal binary16
    b[3, 2:4] = half(-(2.0 ** -22))
    b[4, 4:144] = 255                  # every field 63, every code 15
    b[5, 16:144] = 0                   # every code 0: the min terms alone
    return b


@pytest.mark.parametrize("which", [0, 2])
def test_probe_q4_bit_exact(orc, which):
    """One-hot rows through the projection kernel: column c of each matrix,
    bit for bit the oracle's dequantized weight (decode plan, binary32)."""
    H, I, E = 256, 512, 4
    L = _tiny(orc, E=E, k=1, H=H, I=I)
    nb = H * I // 256
    L["gate"][1] = _edge_blocks(nb, 1)
    L["up"][1] = _edge_blocks(nb, 2)
    L["down"][1] = _edge_blocks(nb, 3)
    lay = _load(L)
    for e in (1, 3):
        K = H if which == 0 else I
        eye = torch.eye(K, device="cuda")
        out = torch.empty(K, 2 * I if which == 0 else H, dtype=torch.float32, device="cuda")
        for r0 in range(0, K, 8):
            m.ds4moe_probe(lay.h, 0, which, e, eye[r0:r0 + 8], out[r0:r0 + 8])
        torch.cuda.synchronize()
        assert m.ds4moe_get_device_error(lay.h) == 0
        if which == 0:
            ref = np.concatenate([orc.dequant_q4k(L[n][e].numpy()).reshape(I, H) for n in ("gate", "up")]).T
        else:
            ref = orc.dequant_q4k(L["down"][e].numpy()).reshape(H, I).T
        got = out.cpu().numpy()
        a = (np.ascontiguousarray(got, np.float32) + np.float32(0)).view(np.uint32)
        b = (np.ascontiguousarray(ref, np.float32) + np.float32(0)).view(np.uint32)
        bad = np.flatnonzero(a != b)
        assert bad.size == 0, (e, bad.size, np.unravel_index(bad[0], a.shape))


# ------------------------------------------------------------------ forward
@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_forward_q4_tiny_matches_oracle(orc, n):
    L = _tiny(orc)
    lay = _load(L)
    x = synth.tokens(n, 256, seed=30 + n)
    out = lay.forward(x.cuda()).cpu().numpy()
    ref, _, _ = orc.moe_forward(oracle_layer(L), x.numpy())
    assert rel_err(out, ref) < TOL


@pytest.mark.parametrize("variant", ["bias", "no_shared", "one_expert", "bf16_act", "wide_hidden", "residual"])
def test_forward_q4_variants(orc, variant):
    kw = dict(bias=variant == "bias", shared=variant != "no_shared")
    if variant == "one_expert":
        kw.update(E=1, k=1)
    if variant == "wide_hidden":   # several routed chunks per task and superblocks per stage
        kw.update(H=1024, I=512)
    L = _tiny(orc, **kw)
    act = m.DS4MOE_ACT_BF16 if variant == "bf16_act" else m.DS4MOE_ACT_F32
    lay = _load(L, act=act)
    n = 3
    x = synth.tokens(n, L["H"], seed=41, dtype=torch.bfloat16 if act else torch.float32)
    out = lay.forward(x.cuda(), residual=variant == "residual").cpu().numpy()
    ref, _, _ = orc.moe_forward(oracle_layer(L), x.float().numpy())
    if variant == "residual":
        ref = ref + x.double().numpy()
    assert rel_err(out, ref) < TOL


@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_forward_q4_full_decode_shape(orc, n):
    """n tokens through a full-size 4-bit layer (H 4096, I 2048, 256 experts top-8, bf16 shared)."""
    L = synth.packed_layer(synth.FULL, 7, device="cuda", expert_bits=4)
    lay = _load(L, max_tokens=8)
    x = synth.tokens(n, 4096, seed=50 + n)
    out = lay.forward(x.cuda()).cpu().numpy()
    ids_gpu, _ = lay.route(x.cuda())
    lg = orc.router_logits(x.numpy(), L["W_r"].cpu().numpy())
    rid, _ = orc.topk_softmax(lg, 8)
    assert np.array_equal(ids_gpu.cpu().numpy(), rid)
    ref, ids, _ = orc.moe_forward(oracle_layer(L, experts=rid.ravel()), x.numpy())
    assert np.array_equal(ids, rid)
    assert rel_err(out, ref) < TOL


def test_forward_q4_full_shape_expert_of_every_token(orc):
    """Eight tokens that all choose expert 17: one expert read by several routed entries."""
    bias = torch.zeros(256)
    bias[17] = 30.0
    L = synth.packed_layer(synth.FULL, 8, bias=bias, device="cuda", expert_bits=4)
    lay = _load(L, max_tokens=8, act=m.DS4MOE_ACT_BF16)
    x = synth.tokens(8, 4096, seed=9, dtype=torch.bfloat16)
    out = lay.forward(x.cuda()).cpu().numpy()
    lg = orc.router_logits(x.float().numpy(), L["W_r"].cpu().numpy(), bias.numpy())
    rid, _ = orc.topk_softmax(lg, 8)
    assert np.all(rid[:, 0] == 17)
    ref, _, _ = orc.moe_forward(oracle_layer(L, experts=rid.ravel()), x.float().numpy())
    assert rel_err(out, ref) < TOL


def test_forward_q4_repeatable(orc):
    L = _tiny(orc)
    lay = _load(L)
    x = synth.tokens(4, 256, seed=7).cuda()
    outs = [lay.forward(x).cpu().numpy() for _ in range(3)]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])



# ------------------------------------------------------------------ tensor-core plan (more than decode_max tokens)
PTOL = 2e-3   # the bf16 reading's bar (x, dequantized weights and h rounded to bf16, fp32 accumulation)


@pytest.mark.parametrize("n", [24, 200])
def test_forward_q4_prefill_tiny_matches_oracle(orc, n):
    L = _tiny(orc)
    lay = _load(L, max_tokens=256, act=m.DS4MOE_ACT_BF16)
    x = synth.tokens(n, 256, seed=80 + n, dtype=torch.bfloat16)
    out = lay.forward(x.cuda()).cpu().numpy()
    ref, _, _ = orc.moe_forward(oracle_layer(L), x.float().numpy(), mode=1)
    assert rel_err(out, ref) < PTOL


@pytest.mark.parametrize("variant", ["f32_act", "no_shared", "bias", "two_row_tiles", "wide_hidden"])
def test_forward_q4_prefill_variants(orc, variant):
    kw = dict(bias=variant == "bias", shared=variant != "no_shared")
    n = 64
    if variant == "two_row_tiles":   # about 300 rows per expert: a full 256-row tile and a ragged one
        kw.update(E=4, k=2)
        n = 600
    if variant == "wide_hidden":
        kw.update(H=1024, I=512)
    L = _tiny(orc, **kw)
    act = m.DS4MOE_ACT_F32 if variant == "f32_act" else m.DS4MOE_ACT_BF16
    lay = _load(L, max_tokens=n, act=act)
    x = synth.tokens(n, L["H"], seed=90, dtype=torch.float32 if act == m.DS4MOE_ACT_F32 else torch.bfloat16)
    out = lay.forward(x.cuda()).cpu().numpy()
    ref, _, _ = orc.moe_forward(oracle_layer(L), x.float().numpy(), mode=1)
    assert rel_err(out, ref) < PTOL


@pytest.mark.parametrize("which", [0, 2])
def test_probe_q4_prefill_bit_exact(orc, which):
    """One-hot bf16 rows through the tensor-core plan's GEMM: column c of each matrix is the oracle's
    dequantized weight rounded to bf16, bit for bit (edge blocks included)."""
    from tests.test_gpu_exact import _probe_columns, _same_bits

    H, I, E = 256, 512, 4
    L = _tiny(orc, E=E, k=1, H=H, I=I)
    nb = H * I // 256
    L["gate"][1] = _edge_blocks(nb, 4)
    L["up"][1] = _edge_blocks(nb, 5)
    L["down"][1] = _edge_blocks(nb, 6)
    lay = _load(L, max_tokens=64)
    for e in (1, 2):
        got = _probe_columns(lay, 1, which, e)
        if which == 0:
            ref = np.concatenate([orc.dequant_q4k(L[n][e].numpy()).reshape(I, H) for n in ("gate", "up")]).T
        else:
            ref = orc.dequant_q4k(L["down"][e].numpy()).reshape(H, I).T
        _same_bits(got, orc.bf16_round(ref))


def test_forward_q4_prefill_full_shape_short_prompt(orc):
    """512 bf16 tokens through a full-size 4-bit layer with Zipf(1.1) expert popularity (sampled outputs)."""
    bias = synth.zipf_bias(256, 1.1, seed=5)
    L = synth.packed_layer(synth.FULL, 6, bias=bias, device="cuda", expert_bits=4)
    n = 512
    lay = _load(L, max_tokens=n, act=m.DS4MOE_ACT_BF16)
    x = synth.tokens(n, 4096, seed=9, dtype=torch.bfloat16)
    out = lay.forward(x.cuda()).cpu().numpy()
    lg = orc.router_logits(x.float().numpy(), L["W_r"].cpu().numpy(), bias.numpy())
    rid, _ = orc.topk_softmax(lg, 8)
    ids, _ = lay.route(x.cuda())
    assert np.array_equal(ids.cpu().numpy(), rid)
    sample = [0, 1, 255, 511]
    ref, _, _ = orc.moe_forward(oracle_layer(L, experts=rid[sample].ravel()), x[sample].float().numpy(), mode=1)
    assert rel_err(out[sample], ref) < PTOL
    assert np.isfinite(out).all()
