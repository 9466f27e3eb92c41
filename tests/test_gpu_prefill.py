"""GPU parity of the prefill (bf16 tensor-core) plan against the CPU oracle, through the C ABI.

Bars: routed expert ids bit-exact (canonical binary32 logits); outputs within
2e-3 of max|ref| against the oracle's bf16 reading (x, dequantized weights and
h rounded to bfloat16 where the tensor-core path rounds them).
"""
import numpy as np
import pytest
import torch

import bit_quantized_moe_softmax_b200 as m
from bit_quantized_moe_softmax_b200 import synth
from tests._util import oracle_layer, pack_with_oracle, rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_moe_softmax_b200 import build

    build.build()


def _tiny(orc, E=8, k=2, seed=0, bias=False, shared=True, router_std=0.02):
    b = synth.zipf_bias(E, 1.1, seed) if bias else None
    L = synth.float_layer(synth.Shape(H=256, I=128, E=E, k=k, shared=shared), seed, router_std=router_std, bias=b)
    L.update(pack_with_oracle(orc, L))
    return L


def _gpu(L, max_tokens, act=m.DS4MOE_ACT_BF16):
    lay = m.MoELayer(L["H"], L["I"], L["E"], L["k"], max_tokens, act_dtype=act,
                     has_shared=L.get("sh_gate") is not None, has_bias=L.get("b_r") is not None)
    lay.load(L)
    return lay


@pytest.mark.parametrize("n", [9, 24, 200])
def test_prefill_tiny_matches_oracle(orc, n):
    L = _tiny(orc)
    lay = _gpu(L, max_tokens=256)
    x = synth.tokens(n, 256, seed=40 + n, dtype=torch.bfloat16)
    out = lay.forward(x.cuda()).cpu().numpy()
    ids, _ = lay.route(x.cuda())
    ref, rid, _ = orc.moe_forward(oracle_layer(L), x.float().numpy(), mode=1)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert rel_err(out, ref) < TOL


@pytest.mark.parametrize("variant", ["f32_act", "no_shared", "bias", "many_rows_per_expert", "one_expert"])
def test_prefill_tiny_variants(orc, variant):
    kw = {}
    n, act = 64, m.DS4MOE_ACT_BF16
    if variant == "f32_act":
        act = m.DS4MOE_ACT_F32
    if variant == "no_shared":
        kw["shared"] = False
    if variant == "bias":
        kw["bias"] = True
    if variant == "many_rows_per_expert":   # ~300 slots per expert: 3 row tiles, ragged tail
        kw.update(E=4, k=2)
        n = 600
    if variant == "one_expert":
        kw.update(E=1, k=1)
        n = 130
    L = _tiny(orc, **kw)
    lay = _gpu(L, max_tokens=1024, act=act)
    x = synth.tokens(n, 256, seed=7, dtype=torch.float32 if act == m.DS4MOE_ACT_F32 else torch.bfloat16)
    out = lay.forward(x.cuda()).cpu().numpy()
    ref, _, _ = orc.moe_forward(oracle_layer(L), x.float().numpy(), mode=1)
    assert rel_err(out, ref) < TOL


def test_prefill_repeatable(orc):
    L = _tiny(orc)
    lay = _gpu(L, max_tokens=256)
    x = synth.tokens(100, 256, seed=3, dtype=torch.bfloat16).cuda()
    a = lay.forward(x).cpu()
    b = lay.forward(x).cpu()
    assert torch.equal(a, b)


def test_prefill_full_shape_short_prompt(orc):
    """512 tokens through a full-size layer with Zipf(1.1) expert popularity (sampled outputs)."""
    bias = synth.zipf_bias(256, 1.1, seed=5)
    L = synth.packed_layer(synth.FULL, 5, bias=bias, device="cuda")
    n = 512
    lay = _gpu(L, max_tokens=n)
    x = synth.tokens(n, 4096, seed=9, dtype=torch.bfloat16)
    out = lay.forward(x.cuda()).cpu().numpy()
    ids, _ = lay.route(x.cuda())
    lg = orc.router_logits(x.float().numpy(), L["W_r"].cpu().numpy(), bias.numpy())
    rid, _ = orc.topk_softmax(lg, 8)
    assert np.array_equal(ids.cpu().numpy(), rid)
    sample = [0, 1, 255, 511]
    need = rid[sample].ravel()
    ref, _, _ = orc.moe_forward(oracle_layer(L, experts=need), x[sample].float().numpy(), mode=1)
    assert rel_err(out[sample], ref) < TOL


def test_prefill_full_shape_long_prompt(orc):
    """The long-prompt workload at full size (11,709 bf16 tokens, Zipf(1.1)), in the launch configuration the
    bench times: routing ids exact for every token, outputs checked on sampled tokens."""
    bias = synth.zipf_bias(256, 1.1, seed=5)
    L = synth.packed_layer(synth.FULL, 7, bias=bias, device="cuda")
    n = 11709
    lay = _gpu(L, max_tokens=n)
    x = synth.tokens(n, 4096, seed=12, dtype=torch.bfloat16)
    out = lay.forward(x.cuda()).cpu().numpy()
    ids, _ = lay.route(x.cuda())
    lg = orc.router_logits(x.float().numpy(), L["W_r"].cpu().numpy(), bias.numpy())
    rid, _ = orc.topk_softmax(lg, 8)
    assert np.array_equal(ids.cpu().numpy(), rid)
    counts = np.bincount(rid.ravel(), minlength=256)
    assert counts.max() > 1000 and (counts < 128).sum() > 100   # the skew the workload is about
    sample = [0, 1, 4096, 8191, n - 2, n - 1]
    need = rid[sample].ravel()
    ref, _, _ = orc.moe_forward(oracle_layer(L, experts=need), x[sample].float().numpy(), mode=1)
    assert rel_err(out[sample], ref) < TOL
    assert np.isfinite(out).all()


# ------------------------------------------------------------------ permutation (counting sort) pins
@pytest.mark.parametrize("n,E,k,zipf", [(40, 8, 2, False), (512, 256, 8, True), (11709, 256, 8, True),
                                        (3000, 1024, 16, True)])
def test_permutation_is_a_stable_counting_sort(n, E, k, zipf):
    """The prefill plan's permutation on routing ids (drawn with the workload's Zipf skew): counts sum to
    n k and equal a histogram, offsets are their exclusive prefix, positions form a permutation, and the
    slots of one expert keep their order -- position for position what numpy's stable argsort gives."""
    g = torch.Generator().manual_seed(n + E)
    if zipf:
        p = torch.exp(synth.zipf_bias(E, 1.1, seed=5).double())
        ids = torch.multinomial(p.expand(n, E), k, replacement=False, generator=g).to(torch.int32)
    else:
        ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(n)]).to(torch.int32)
    lay = m.MoELayer(256, 128, E, k, max_tokens=n + 16)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty(n * k, dtype=torch.int32, device="cuda")
    m.ds4moe_permutation(lay.h, ids.cuda(), counts, offs, pos)
    flat = ids.numpy().ravel()
    ref_counts = np.bincount(flat, minlength=E)
    assert np.array_equal(counts.cpu().numpy(), ref_counts) and ref_counts.sum() == n * k
    assert np.array_equal(offs.cpu().numpy(), np.concatenate([[0], np.cumsum(ref_counts)]))
    p = pos.cpu().numpy()
    assert np.array_equal(np.sort(p), np.arange(n * k))                  # a permutation
    order = np.argsort(flat, kind="stable")                              # slots by expert, slot order kept
    assert np.array_equal(p[order], np.arange(n * k))


# ------------------------------------------------------------------ every token of chosen experts
def _oracle_rows(orc, lay, X):
    """The oracle's bf16 reading of a one-expert layer (E = k = 1) on the rows X, split over the host's
    cores: each thread runs one chunk of rows through one call (the expert dequantized once per chunk)."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    parts = np.array_split(np.arange(X.shape[0]), max(1, min(os.cpu_count() or 1, X.shape[0])))
    with ThreadPoolExecutor(max_workers=len(parts)) as ex:
        outs = list(ex.map(lambda r: orc.moe_forward(lay, X[r], mode=1)[0], parts))
    return np.concatenate(outs, axis=0)


def _one_expert_layer(L, e, shared):
    """Expert e of L as the only expert of a layer (E = k = 1, weight 1), with or without L's shared expert;
    e = None: an all-zero expert (its output is exactly zero), so the layer is the shared expert alone."""
    nb = L["I"] * L["H"] // 256
    sh = oracle_layer(L, experts=[]) if shared else None
    return dict(H=L["H"], I=L["I"], E=1, k=1, W_r=np.zeros((1, L["H"]), np.float32), b_r=None,
                grid=L["grid"].cpu().numpy(),
                gate=[np.zeros((nb, 66), np.uint8) if e is None else L["gate"][e].cpu().numpy()],
                up=[np.zeros((nb, 66), np.uint8) if e is None else L["up"][e].cpu().numpy()],
                down=[np.zeros((nb, 84), np.uint8) if e is None else L["down"][e].cpu().numpy()],
                sh_gate=sh["sh_gate"] if shared else None, sh_up=sh["sh_up"] if shared else None,
                sh_down=sh["sh_down"] if shared else None)


@pytest.mark.parametrize("n", [512, 11709])
def test_prefill_every_token_of_chosen_experts(orc, n):
    """The prefill workloads at full size: the outputs of the tokens routed to the most popular expert
    (two tokens of each 256-row tile and every token of its ragged last tile), to the least chosen
    expert and to one with 129..255 tokens, against the oracle.  Every other expert's down
    matrix is zero, so a token's output is the shared expert plus the weighted outputs of the chosen
    experts it selected, and the oracle needs only those three experts.  (The least chosen expert has
    fewer than 16 tokens at 512 tokens and about 46 at 11,709.)"""
    bias = synth.zipf_bias(256, 1.1, seed=5)
    L = synth.packed_layer(synth.FULL, 7, bias=bias, device="cuda")
    x = synth.tokens(n, 4096, seed=12, dtype=torch.bfloat16)
    lg = orc.router_logits(x.float().numpy(), L["W_r"].cpu().numpy(), bias.numpy())
    rid, rw = orc.topk_softmax(lg, 8)
    counts = np.bincount(rid.ravel(), minlength=256)
    top = int(np.argmax(counts))
    small = int(np.flatnonzero(counts == counts[counts > 0].min())[0])   # the least chosen (< 16 at 512 tokens)
    mids = np.flatnonzero((counts > 128) & (counts < 256))
    chosen = [top, small] + ([int(mids[0])] if mids.size else [])
    down = L["down"].clone()
    keep = torch.zeros(256, dtype=torch.bool)
    keep[chosen] = True
    down[~keep.to(down.device), :, 80:84] = 0          # d = dmin = 0: every other expert's down weights are 0
    L["down"] = down
    lay = _gpu(L, max_tokens=n)
    out = lay.forward(x.cuda()).cpu().numpy()
    # the tokens to check: the popular expert's rows in permuted (slot) order, two per tile and the whole tail
    slots = np.flatnonzero(rid.ravel() == top)
    picks = []
    for t0 in range(0, slots.size, 256):
        tile = slots[t0:t0 + 256]
        picks += list(tile) if t0 + 256 >= slots.size else [tile[0], tile[-1]]
    toks = sorted(set(int(s) // 8 for s in picks) | set(int(s) // 8 for e in chosen[1:] for s in
                                                        np.flatnonzero(rid.ravel() == e)))
    X = x.float().numpy()[toks]
    ref = _oracle_rows(orc, _one_expert_layer(L, None, shared=True), X)
    for e in chosen:
        rows = [i for i, t in enumerate(toks) if e in rid[t]]
        ye = _oracle_rows(orc, _one_expert_layer(L, e, shared=False), X[rows])
        for r, i in enumerate(rows):
            j = int(np.flatnonzero(rid[toks[i]] == e)[0])
            ref[i] += rw[toks[i], j] * ye[r]
    assert rel_err(out[toks], ref) < TOL
