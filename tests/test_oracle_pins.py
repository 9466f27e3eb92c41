"""Pins for the CPU oracle: each check ties it to something other than itself.

Closed forms for hand-built blocks, library routines for the number formats
(numpy's binary16, torch's bfloat16), exact integer arithmetic and brute-force
sorting for the router, and invariants of the layer (identical experts
collapse to one dense FFN, a zero routed part leaves the shared expert, expert
relabelling changes nothing) that reduce the whole forward to a textbook dense
FFN evaluated with numpy / torch.
"""
import math

import numpy as np
import pytest
import torch

from bit_quantized_moe_softmax_b200 import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ----------------------------------------------------------------- formats
def test_half_to_double_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.half_to_double(int(b)) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_double_to_half_matches_numpy(orc):
    rng = np.random.default_rng(0)
    vals = list(rng.standard_normal(4000) * 10.0 ** rng.integers(-9, 5, 4000))
    # exact ties between neighbouring halves, subnormal ties, overflow edges
    h = np.arange(0, 0x7c00, 97, dtype=np.uint16).view(np.float16).astype(np.float64)
    hn = (np.arange(0, 0x7c00, 97, dtype=np.uint16) + 1).view(np.float16).astype(np.float64)
    vals += list((h + hn) / 2) + list(-(h + hn) / 2)
    vals += [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -25, 2.0 ** -24 * 1.5, 2.0 ** -26]
    for v in vals:
        assert orc.double_to_half(v) == int(np.array(v, dtype=np.float64).astype(np.float16).view(np.uint16)), v


def test_bf16_round_matches_torch(orc):
    rng = np.random.default_rng(1)
    v = (rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000)).astype(np.float32)
    # exact ties: low 16 bits == 0x8000, both parities of bit 16
    u = rng.integers(0, 2 ** 31, 1000, dtype=np.uint64).astype(np.uint32)
    ties = ((u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    ties = ties[np.isfinite(ties)]
    v = np.concatenate([v, ties, np.array([1e-40, -1e-42, 3.3e38], dtype=np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(orc.bf16_round(v), ref)


def _q2_handbuilt():
    """d = 1.0, dmin = 0.5, sc_j = j, m_j = 15 - j, q_i = i mod 4."""
    b = np.zeros(84, dtype=np.uint8)
    for j in range(16):
        b[j] = j | ((15 - j) << 4)
    for i in range(256):
        b[16 + i // 4] |= (i % 4) << (2 * (i % 4))
    b[80:82] = [0x00, 0x3C]
    b[82:84] = [0x00, 0x38]
    return b


def test_q2k_dequant_closed_form(orc):
    out = orc.dequant_q2k(_q2_handbuilt())
    i = np.arange(256)
    j = i // 16
    assert np.array_equal(out, (j * (i % 4) - 0.5 * (15 - j)).astype(np.float32))


def test_q2k_dequant_single_fields(orc):
    # one code, one scale, one min, d and dmin each moved on their own
    base = np.zeros(84, dtype=np.uint8)
    base[80:82] = [0x00, 0x40]   # d = 2
    base[82:84] = [0x00, 0x34]   # dmin = 0.25
    b = base.copy()
    b[5] = 3 | (7 << 4)          # sub-block 5: sc = 3, m = 7
    b[16 + 83 // 4] |= 2 << (2 * (83 % 4))   # weight 83 (sub-block 5) q = 2
    out = orc.dequant_q2k(b)
    exp = np.zeros(256, dtype=np.float32)
    exp[80:96] = -0.25 * 7
    exp[83] = 2 * 3 * 2 - 0.25 * 7
    assert np.array_equal(out, exp)
    # two blocks back to back keep their own fields
    two = np.concatenate([_q2_handbuilt(), b])
    out2 = orc.dequant_q2k(two)
    assert np.array_equal(out2[256:], exp)


def test_q2k_dequant_rounds_once_to_binary32(orc):
    # d*sc*q - dmin*m with d, dmin far apart: exact value needs > 24 bits
    b = np.zeros(84, dtype=np.uint8)
    b[0] = 15 | (15 << 4)
    b[16] = 3
    dh = np.array(1.0 + 2.0 ** -10, dtype=np.float16).view(np.uint16)
    mh = np.array(2.0 ** -24, dtype=np.float16).view(np.uint16)
    b[80:82] = [int(dh) & 0xFF, int(dh) >> 8]
    b[82:84] = [int(mh) & 0xFF, int(mh) >> 8]
    out = orc.dequant_q2k(b)
    exact = 45 * (1.0 + 2.0 ** -10) - 15 * 2.0 ** -24
    assert out[0] == np.float32(exact)
    assert out[1] == np.float32(-15 * 2.0 ** -24)


# ---------------------------------------------------------------- Q4_K-style (4-bit experts)
def _q4_block(d, dmin, sc, m, q):
    """144-byte block written from the layout: d, dmin binary16; sixteen 6-bit
    fields (sc_0..7 then m_0..7) packed little-endian into bytes 4..15; codes
    two per byte, low nibble first."""
    b = np.zeros(144, dtype=np.uint8)
    b[0:2] = np.frombuffer(np.array(d, np.float16).tobytes(), np.uint8)
    b[2:4] = np.frombuffer(np.array(dmin, np.float16).tobytes(), np.uint8)
    fields = 0
    for f, v in enumerate(list(sc) + list(m)):
        fields |= int(v) << (6 * f)
    b[4:16] = np.frombuffer(fields.to_bytes(12, "little"), np.uint8)
    for i in range(256):
        b[16 + i // 2] |= int(q[i]) << (4 * (i % 2))
    return b


def test_q4k_dequant_closed_form(orc):
    i = np.arange(256)
    j = i // 32
    sc, m = 8 * np.arange(8) + 7, 63 - 8 * np.arange(8)
    out = orc.dequant_q4k(_q4_block(1.0, 0.5, sc, m, i % 16))
    assert np.array_equal(out, (sc[j] * (i % 16) - 0.5 * m[j]).astype(np.float32))


def test_q4k_field_bytes(orc):
    # single fields set at the byte level: bit 6 of byte 4 is sc_1's lowest bit,
    # bit 0 of byte 10 (bit 48) is m_0's, bits 2..7 of byte 15 (90..95) are m_7
    b = np.zeros(144, dtype=np.uint8)
    b[0:2] = [0x00, 0x40]            # d = 2
    b[2:4] = [0x00, 0x34]            # dmin = 0.25
    b[4] = 0x40                      # sc_1 = 1
    b[10] = 0x01                     # m_0 = 1
    b[15] = 0xFC                     # m_7 = 63
    b[16:144] = 0x33                 # every code 3
    b[16] = 0x21                     # q_0 = 1, q_1 = 2
    out = orc.dequant_q4k(b)
    exp = np.zeros(256, dtype=np.float32)
    exp[0:32] = -0.25
    exp[0], exp[1] = 2 * 0 * 1 - 0.25, 2 * 0 * 2 - 0.25
    exp[32:64] = 2 * 1 * 3
    exp[224:256] = -0.25 * 63
    assert np.array_equal(out, exp)
    # a second block after it keeps its own fields
    two = orc.dequant_q4k(np.concatenate([_q4_block(1.0, 0.5, [1] * 8, [0] * 8, np.full(256, 15)), b]))
    assert np.array_equal(two[:256], np.full(256, 15, np.float32)) and np.array_equal(two[256:], exp)


def test_q4k_pack_exact_roundtrip(orc):
    # codes 0..15 times step = 63 * 2^-6, no negatives: d = 2^-6, sc = 63, dmin = 0
    rng = np.random.default_rng(7)
    step = 63 * 2.0 ** -6
    q = rng.integers(0, 16, (3, 256))
    q[:, ::32] = 15
    w = (q * step).astype(np.float32)
    blocks = orc.pack_q4k(w)
    assert blocks.shape == (3, 144)
    assert np.array_equal(orc.dequant_q4k(blocks), w.ravel())
    assert all(bytes(bl[0:2]) == np.array(2.0 ** -6, np.float16).tobytes() for bl in blocks)
    assert np.all(blocks[:, 2:4] == 0)
    assert np.array_equal(blocks[0], _q4_block(2.0 ** -6, 0.0, [63] * 8, [0] * 8, q[0]))


def test_q4k_pack_zero_error_and_finer_than_q2k(orc):
    assert not orc.pack_q4k(np.zeros(512, np.float32)).any()
    with pytest.raises(ValueError):
        orc.pack_q4k(np.zeros(300, np.float32))
    rng = np.random.default_rng(8)
    w = (rng.standard_normal(256 * 64) * 0.02).astype(np.float32)
    r4 = orc.dequant_q4k(orc.pack_q4k(w))
    r2 = orc.dequant_q2k(orc.pack_q2k(w))
    e4 = np.sqrt(np.mean((r4 - w) ** 2)) / np.std(w)
    e2 = np.sqrt(np.mean((r2 - w) ** 2)) / np.std(w)
    assert e4 < 0.1 and e4 < e2 / 3, (e4, e2)   # 4.5 bits per weight against 2.6
    # error of each weight: half a code step, plus what rounding the fields
    # costs -- sc_j off by <= 1/2 (times 15 steps of d) and m_j by <= 1/2 (of dmin)
    for blk, wb in zip(orc.pack_q4k(w), w.reshape(-1, 256)):
        d = float(np.frombuffer(blk[0:2].tobytes(), np.float16)[0])
        dmin = float(np.frombuffer(blk[2:4].tobytes(), np.float16)[0])
        fields = int.from_bytes(blk[4:16].tobytes(), "little")
        sc = [(fields >> (6 * j)) & 63 for j in range(8)]
        dq = orc.dequant_q4k(blk).astype(np.float64)
        for j in range(8):
            s = slice(32 * j, 32 * j + 32)
            bound = 0.5 * d * sc[j] + 7.5 * d + 0.5 * dmin
            assert np.all(np.abs(dq[s] - wb[s]) <= bound * (1 + 1e-6))


def _iq2_block(d_bits, groups):
    """groups: list of 8 tuples (indices[4], sigmas[4], s)."""
    b = np.zeros(66, dtype=np.uint8)
    b[0:2] = [d_bits & 0xFF, d_bits >> 8]
    for g, (idx, sig, s) in enumerate(groups):
        S = s << 28
        for c in range(4):
            b[2 + 8 * g + c] = idx[c]
            S |= sig[c] << (7 * c)
        b[2 + 8 * g + 4: 2 + 8 * g + 8] = np.frombuffer(np.uint32(S).tobytes(), dtype=np.uint8)
    return b


def test_iq2_dequant_closed_form(orc):
    grid = np.full((256, 8), 8, dtype=np.uint8)
    grid[0] = [8, 25, 43, 8, 25, 43, 8, 25]
    grid[5] = [43, 43, 8, 8, 25, 25, 43, 8]
    zero = ([0, 0, 0, 0], [0, 0, 0, 0], 0)
    groups = [zero] * 8
    groups[0] = ([0, 0, 0, 0], [0, 1, 0x7F, 0b0000011], 0)
    groups[3] = ([5, 0, 0, 0], [0, 0, 0, 0], 15)
    out = orc.dequant_iq2xxs(_iq2_block(0x3C00, groups), grid)   # d = 1.0
    r0 = np.array([8, 25, 43, 8, 25, 43, 8, 25]) / 8.0
    assert np.array_equal(out[0:8], r0)                                  # sigma 0: all +
    assert np.array_equal(out[8:16], r0 * [-1, 1, 1, 1, 1, 1, 1, -1])   # bit 0 + parity
    assert np.array_equal(out[16:24], -r0)                               # 7 bits: odd -> 8th too
    assert np.array_equal(out[24:32], r0 * [-1, -1, 1, 1, 1, 1, 1, 1])  # 2 bits: even
    r5 = np.array([43, 43, 8, 8, 25, 25, 43, 8]) * 31 / 8.0             # s = 15 -> (2s+1)/8
    assert np.array_equal(out[96:104], r5)
    assert np.array_equal(out[104:128], np.tile(r0 * 31, 3))           # chunks 1..3: row 0
    assert np.array_equal(out[32:96], np.tile(r0, 8))                   # groups 1, 2: row 0, s 0


def test_iq2_dequant_scale_and_d(orc):
    grid = synth.grid_table(0).numpy()
    rng = np.random.default_rng(3)
    groups = [(list(rng.integers(0, 256, 4)), [0, 0, 0, 0], int(s)) for s in range(8)]
    d = np.float16(0.00347)
    out = orc.dequant_iq2xxs(_iq2_block(int(np.array(d).view(np.uint16)), groups), grid)
    for g, (idx, _, s) in enumerate(groups):
        for c in range(4):
            exp = float(d) * (2 * s + 1) / 8 * grid[idx[c]].astype(np.float64)
            assert np.array_equal(out[32 * g + 8 * c: 32 * g + 8 * c + 8], exp.astype(np.float32))


# ----------------------------------------------------------------- packers
def test_q2k_pack_exact_roundtrip(orc):
    # each sub-block holds the codes 0..3 times a = 15 * 2^-6, no negative values:
    # d = 2^-6, sc = 15, dmin = 0 and the codes come back exactly
    rng = np.random.default_rng(4)
    a = 15 * 2.0 ** -6
    q = rng.integers(0, 4, (3, 256))
    q[:, ::16] = 3
    w = (q * a).astype(np.float32)
    blocks = orc.pack_q2k(w)
    assert np.array_equal(orc.dequant_q2k(blocks), w.ravel())
    assert all(bytes(b[80:82]) == bytes(np.array(2.0 ** -6, np.float16).tobytes()) for b in blocks)
    assert np.all(blocks[:, 82:84] == 0)


def test_q2k_pack_zero_and_error(orc):
    z = orc.pack_q2k(np.zeros(512, np.float32))
    assert not z.any()
    rng = np.random.default_rng(5)
    w = (rng.standard_normal(256 * 64) * 0.02).astype(np.float32)
    r = orc.dequant_q2k(orc.pack_q2k(w))
    rel = np.sqrt(np.mean((r - w) ** 2)) / np.std(w)
    assert rel < 0.35, rel      # 2.6 bits per weight
    # codes/scales are in range and every sub-block's value range spans its data
    for blk, wb in zip(orc.pack_q2k(w).reshape(-1, 84), w.reshape(-1, 256)):
        dq = orc.dequant_q2k(blk)
        for j in range(16):
            s = slice(16 * j, 16 * j + 16)
            assert dq[s].min() <= max(0.0, wb[s].min()) + 1e-2


def test_iq2_pack_exact_roundtrip(orc):
    grid = synth.grid_table(0).numpy()
    rows43 = [a for a in range(256) if 43 in grid[a]]
    rng = np.random.default_rng(6)
    d = 2.0 ** -8
    db = d * 31 / 8
    w = np.zeros((2, 256))
    expect_idx = []
    for b in range(2):
        for g in range(8):
            for c in range(4):
                a = int(rows43[rng.integers(len(rows43))]) if c == 0 else int(rng.integers(256))
                neg = rng.integers(0, 2, 8)
                if neg.sum() % 2:
                    neg[7] ^= 1
                w[b, 32 * g + 8 * c: 32 * g + 8 * c + 8] = db * grid[a] * np.where(neg, -1, 1)
                expect_idx.append(a)
    blocks = orc.pack_iq2xxs(w.astype(np.float32), grid)
    assert np.array_equal(orc.dequant_iq2xxs(blocks, grid), w.ravel().astype(np.float32))
    got_idx = [int(blocks[b, 2 + 8 * g + c]) for b in range(2) for g in range(8) for c in range(4)]
    assert got_idx == expect_idx


def test_iq2_pack_sign_parity_and_zero(orc):
    grid = synth.grid_table(0).numpy()
    assert not orc.pack_iq2xxs(np.zeros(256, np.float32), grid).any()
    w = np.full(256, 0.01, dtype=np.float32)
    w[0:8] = [-0.01, 0.02, 0.03, 0.04, 0.05, 0.06, 0.07, 0.005]   # one negative: odd
    blk = orc.pack_iq2xxs(w, grid)[0]
    S = int(np.frombuffer(blk[6:10].tobytes(), dtype=np.uint32)[0])
    sigma0 = S & 0x7F
    # the smallest magnitude (element 7) is flipped negative; element 0 stays negative
    assert sigma0 == 1
    dq = orc.dequant_iq2xxs(blk, grid)
    assert dq[0] < 0 and dq[7] < 0 and np.all(dq[1:7] > 0)


def test_iq2_pack_error(orc):
    grid = synth.grid_table(0).numpy()
    rng = np.random.default_rng(7)
    w = (rng.standard_normal(256 * 32) * 0.02).astype(np.float32)
    r = orc.dequant_iq2xxs(orc.pack_iq2xxs(w, grid), grid)
    rel = np.sqrt(np.mean((r - w) ** 2)) / np.std(w)
    assert rel < 0.75, rel       # a 3-magnitude random codebook: coarse but bounded


def test_grid_table_distinct():
    g = synth.grid_table(0).numpy()
    assert g.shape == (256, 8)
    assert set(np.unique(g)) <= {8, 25, 43}
    assert len({tuple(r) for r in g}) == 256


# ----------------------------------------------------------------- router
def test_router_logit_exact_integers(orc):
    rng = np.random.default_rng(8)
    x = rng.integers(-8, 9, (3, 256)).astype(np.float32)
    W = rng.integers(-8, 9, (5, 256)).astype(np.float32)
    ref = x.astype(np.int64) @ W.astype(np.int64).T
    assert np.array_equal(orc.router_logits(x, W), ref.astype(np.float32))


def test_router_logit_canonical_order(orc):
    # lane 0's chain holds 2^24 first, so its three following +1 are each lost
    # (ties to even); lane 1's chain keeps four +1; the butterfly adds them.
    x = np.zeros(256, np.float32)
    w = np.ones(256, np.float32)
    x[0] = 2.0 ** 24
    x[1:4] = 1.0
    x[4:8] = 1.0
    assert orc.router_logits(x[None], w[None])[0, 0] == np.float32(2 ** 24 + 4)
    # the second sweep (i = 1) of lane 0 comes after its first sweep
    x2 = np.zeros(256, np.float32)
    x2[1:4] = 1.0
    x2[128] = 2.0 ** 24
    assert orc.router_logits(x2[None], w[None])[0, 0] == np.float32(2 ** 24 + 4)
    # butterfly: p_0 + p_16 first, so 2^24 + 1 + 1 loses both ones
    x3 = np.zeros(256, np.float32)
    x3[0] = 2.0 ** 24
    x3[64] = 1.0        # lane 16
    x3[4 * 8] = 1.0     # lane 8
    assert orc.router_logits(x3[None], w[None])[0, 0] == np.float32(2 ** 24)
    # bias is one binary32 add at the end
    b = np.array([0.5], np.float32)
    assert orc.router_logits(x[None], w[None], b)[0, 0] == np.float32(2 ** 24 + 4)


def test_router_logit_error_bound(orc):
    rng = np.random.default_rng(9)
    H = 4096
    x = rng.standard_normal((4, H)).astype(np.float32)
    W = (rng.standard_normal((16, H)) * 0.02).astype(np.float32)
    b = rng.standard_normal(16).astype(np.float32)
    l32 = orc.router_logits(x, W, b).astype(np.float64)
    l64 = x.astype(np.float64) @ W.astype(np.float64).T + b
    absum = np.abs(x.astype(np.float64)) @ np.abs(W.astype(np.float64)).T + np.abs(b)
    gamma = (H // 32 + 6) * 2.0 ** -24 * 1.01
    assert np.all(np.abs(l32 - l64) <= gamma * absum)
    assert np.allclose(orc.router_logits_f64(x, W, b), l64, rtol=0, atol=1e-12)


def test_topk_brute_force(orc):
    rng = np.random.default_rng(10)
    for E, k in [(8, 2), (256, 8), (16, 16), (1, 1)]:
        lg = rng.integers(-3, 4, (50, E)).astype(np.float32)  # many ties
        lg[:25] += rng.standard_normal((25, E)).astype(np.float32)
        ids, w = orc.topk_softmax(lg, k)
        for t in range(50):
            order = np.lexsort((np.arange(E), -lg[t].astype(np.float64)))
            assert list(ids[t]) == list(order[:k])
        assert np.allclose(w.sum(1), 1.0, rtol=0, atol=1e-12)
        assert np.all(np.diff(w, axis=1) <= 1e-15)


def test_softmax_two_experts_is_logistic(orc):
    from scipy.special import expit

    lg = np.array([[0.3, -1.2], [2.0, 2.0], [-0.5, 4.0]], np.float32)
    ids, w = orc.topk_softmax(lg, 2)
    for t in range(3):
        a, b = lg[t, ids[t, 0]], lg[t, ids[t, 1]]
        assert abs(w[t, 0] - expit(float(a) - float(b))) < 1e-15
    assert list(ids[1]) == [0, 1]


# ----------------------------------------------------------------- layer
def _dense_ffn(Wg, Wu, Wd, x):
    """Textbook SwiGLU FFN through torch library routines, fp64."""
    X = torch.from_numpy(np.asarray(x, np.float64))
    g = X @ torch.from_numpy(np.asarray(Wg, np.float64)).T
    u = X @ torch.from_numpy(np.asarray(Wu, np.float64)).T
    return (torch.nn.functional.silu(g) * u @ torch.from_numpy(np.asarray(Wd, np.float64)).T).numpy()


def _bf16_f64(t):
    return t.to(torch.float32).numpy().astype(np.float64)


def _packed_tiny(orc, E=8, k=2, seed=0, identical=False, zero_routed=False):
    L = synth.float_layer(synth.Shape(H=256, I=128, E=E, k=k), seed)
    grid = L["grid"].numpy()
    lay = dict(H=256, I=128, E=E, k=k, W_r=L["W_r"].numpy(), b_r=None, grid=grid)
    src = 0 if identical else None
    gate, up, down = [], [], []
    for e in range(E):
        s = e if src is None else src
        gf, uf, df = (L[n][s].numpy() for n in ("gate_f", "up_f", "down_f"))
        if zero_routed:
            gf, uf, df = gf * 0, uf * 0, df * 0
        gate.append(orc.pack_iq2xxs(gf, grid))
        up.append(orc.pack_iq2xxs(uf, grid))
        down.append(orc.pack_q2k(df))
    lay.update(gate=gate, up=up, down=down)
    for n in ("sh_gate", "sh_up", "sh_down"):
        lay[n] = L[n].view(torch.int16).numpy().view(np.uint16)
    return lay, L


def test_identical_experts_collapse_to_dense_ffn(orc):
    lay, L = _packed_tiny(orc, identical=True)
    x = synth.tokens(6, 256, seed=1).numpy()
    out, ids, w = orc.moe_forward(lay, x)
    grid = lay["grid"]
    Wg = orc.dequant_iq2xxs(lay["gate"][0], grid).reshape(128, 256)
    Wu = orc.dequant_iq2xxs(lay["up"][0], grid).reshape(128, 256)
    Wd = orc.dequant_q2k(lay["down"][0]).reshape(256, 128)
    ref = _dense_ffn(Wg, Wu, Wd, x) + _dense_ffn(_bf16_f64(L["sh_gate"]), _bf16_f64(L["sh_up"]),
                                                 _bf16_f64(L["sh_down"]), x)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.allclose(w.sum(1), 1.0, atol=1e-12)


def test_identical_q4_experts_collapse_to_dense_ffn(orc):
    """The 4-bit variant: every expert the same Q4_K-style blocks (gate, up and
    down), so the layer is one dense SwiGLU FFN of those weights plus the shared
    expert, evaluated with torch; different experts' blocks change the output."""
    L = synth.float_layer(synth.Shape(H=256, I=128, E=8, k=2), 3)
    blocks = {n: orc.pack_q4k(L[n + "_f"][0].numpy()) for n in ("gate", "up", "down")}
    lay = dict(H=256, I=128, E=8, k=2, W_r=L["W_r"].numpy(), b_r=None, grid=L["grid"].numpy(),
               gate=[blocks["gate"]] * 8, up=[blocks["up"]] * 8, down=[blocks["down"]] * 8, expert_bits=4)
    for n in ("sh_gate", "sh_up", "sh_down"):
        lay[n] = L[n].view(torch.int16).numpy().view(np.uint16)
    x = synth.tokens(6, 256, seed=2).numpy()
    out, ids, w = orc.moe_forward(lay, x)
    Wg = orc.dequant_q4k(blocks["gate"]).reshape(128, 256)
    Wu = orc.dequant_q4k(blocks["up"]).reshape(128, 256)
    Wd = orc.dequant_q4k(blocks["down"]).reshape(256, 128)
    ref = _dense_ffn(Wg, Wu, Wd, x) + _dense_ffn(_bf16_f64(L["sh_gate"]), _bf16_f64(L["sh_up"]),
                                                 _bf16_f64(L["sh_down"]), x)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # other down blocks give another output (the 4-bit blocks are what is read);
    # a bit width other than 2 or 4 is refused
    lay2 = dict(lay, down=[orc.pack_q4k(L["down_f"][1].numpy())] * 8)
    assert not np.allclose(orc.moe_forward(lay2, x)[0], out)
    with pytest.raises(ValueError):
        orc.moe_forward(dict(lay, expert_bits=3), x)


def test_chain_of_dense_layers(orc):
    # two layers whose routed experts are identical: each layer is x + two dense
    # FFNs (routed weights sum to 1, plus the shared expert), computed with torch
    lays = [_packed_tiny(orc, identical=True, seed=s) for s in (0, 5)]
    x = synth.tokens(3, 256, seed=6).numpy()
    got, ids, inputs = orc.chain_forward([lay for lay, _ in lays], x)
    cur = x.astype(np.float32)
    for lay, L in lays:
        grid = lay["grid"]
        Wg = orc.dequant_iq2xxs(lay["gate"][0], grid).reshape(128, 256)
        Wu = orc.dequant_iq2xxs(lay["up"][0], grid).reshape(128, 256)
        Wd = orc.dequant_q2k(lay["down"][0]).reshape(256, 128)
        xd = cur.astype(np.float64)
        y = _dense_ffn(Wg, Wu, Wd, xd) + _dense_ffn(_bf16_f64(L["sh_gate"]), _bf16_f64(L["sh_up"]),
                                                    _bf16_f64(L["sh_down"]), xd)
        cur = (xd + y).astype(np.float32)
    assert len(ids) == 2 and np.array_equal(inputs[0], x.astype(np.float32))
    assert np.abs(got.astype(np.float64) - cur).max() <= 2 ** -20 * np.abs(cur).max()


def test_chain_of_zero_layers_is_identity(orc):
    lay, _ = _packed_tiny(orc, zero_routed=True)
    for n in ("sh_gate", "sh_up", "sh_down"):
        lay[n] = None
    x = synth.tokens(2, 256, seed=7).numpy()
    got, _, _ = orc.chain_forward([lay, lay, lay], x)
    assert np.array_equal(got, x.astype(np.float32))


def test_steer_closed_forms(orc):
    rng = np.random.default_rng(0)
    y = rng.standard_normal((5, 64))
    v = rng.standard_normal(64).astype(np.float32)
    v = (v / np.linalg.norm(v.astype(np.float64))).astype(np.float32)
    vd = v.astype(np.float64)
    for F in (0.0, 0.3, 1.0, 2.5):
        ys = orc.steer(y, v, F)
        nv = vd @ vd   # 1 up to the binary32 rounding of v
        # the component along v scales by 1 - F |v|^2; the orthogonal part is unchanged
        assert np.allclose(ys @ vd, (1 - F * nv) * (y @ vd), rtol=0, atol=1e-12)
        perp = lambda a: a - np.outer(a @ vd, vd) / nv
        assert np.allclose(perp(ys), perp(y), rtol=0, atol=1e-12)
    assert np.array_equal(orc.steer(y, v, 0.0), y)


def test_zero_routed_leaves_shared(orc):
    lay, L = _packed_tiny(orc, zero_routed=True)
    x = synth.tokens(3, 256, seed=2).numpy()
    out, _, _ = orc.moe_forward(lay, x)
    ref = _dense_ffn(_bf16_f64(L["sh_gate"]), _bf16_f64(L["sh_up"]), _bf16_f64(L["sh_down"]), x)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_two_experts_weighted_sum(orc):
    # E = k = 2, distinct experts, no shared expert: out = w0 FFN_id0 + w1 FFN_id1
    lay, L = _packed_tiny(orc, E=2, k=2, seed=3)
    for n in ("sh_gate", "sh_up", "sh_down"):
        lay[n] = None
    x = synth.tokens(4, 256, seed=4).numpy()
    out, ids, w = orc.moe_forward(lay, x)
    grid = lay["grid"]
    ffn = []
    for e in range(2):
        Wg = orc.dequant_iq2xxs(lay["gate"][e], grid).reshape(128, 256)
        Wu = orc.dequant_iq2xxs(lay["up"][e], grid).reshape(128, 256)
        Wd = orc.dequant_q2k(lay["down"][e]).reshape(256, 128)
        ffn.append(_dense_ffn(Wg, Wu, Wd, x))
    lg = orc.router_logits(x, lay["W_r"]).astype(np.float64)   # canonical logits (pinned above)
    from scipy.special import expit

    for t in range(4):
        p0 = expit(lg[t, 0] - lg[t, 1])
        ref = p0 * ffn[0][t] + (1 - p0) * ffn[1][t]
        assert np.allclose(out[t], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_single_expert(orc):
    lay, L = _packed_tiny(orc, E=1, k=1, seed=5)
    x = synth.tokens(2, 256, seed=6).numpy()
    out, ids, w = orc.moe_forward(lay, x)
    assert np.all(ids == 0) and np.all(w == 1.0)
    grid = lay["grid"]
    Wg = orc.dequant_iq2xxs(lay["gate"][0], grid).reshape(128, 256)
    Wu = orc.dequant_iq2xxs(lay["up"][0], grid).reshape(128, 256)
    Wd = orc.dequant_q2k(lay["down"][0]).reshape(256, 128)
    ref = _dense_ffn(Wg, Wu, Wd, x) + _dense_ffn(_bf16_f64(L["sh_gate"]), _bf16_f64(L["sh_up"]),
                                                 _bf16_f64(L["sh_down"]), x)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_expert_relabelling_invariance(orc):
    lay, _ = _packed_tiny(orc, seed=7)
    x = synth.tokens(5, 256, seed=8).numpy()
    out, ids, w = orc.moe_forward(lay, x)
    perm = np.random.default_rng(11).permutation(8)
    lay2 = dict(lay)
    lay2["W_r"] = lay["W_r"][perm]
    for n in ("gate", "up", "down"):
        lay2[n] = [lay[n][p] for p in perm]
    out2, ids2, w2 = orc.moe_forward(lay2, x)
    assert np.array_equal(out, out2)
    assert np.array_equal(perm[ids2], ids)


def test_bf16_reading_close_to_fp64(orc):
    lay, _ = _packed_tiny(orc, seed=9)
    x = synth.tokens(4, 256, seed=10, dtype=torch.bfloat16).float().numpy()
    out0, ids0, _ = orc.moe_forward(lay, x, mode=0)
    out1, ids1, _ = orc.moe_forward(lay, x, mode=1)
    assert np.array_equal(ids0, ids1)
    rel = np.abs(out1 - out0).max() / np.abs(out0).max()
    assert 0 < rel < 2e-2, rel


def test_bf16_reading_exact_when_representable(orc):
    # weights whose dequantized values fit bfloat16 (d a power of two, s = 0,
    # dmin = 0) and bf16 x: the bf16 reading differs from fp64 only through the
    # rounding of h.  With the shared expert off and h forced to tiny magnitudes
    # the rounding of h is the only source; check it is bounded by 2^-8 relative.
    grid = synth.grid_table(0).numpy()
    rng = np.random.default_rng(12)
    H, I = 256, 128
    iq = np.zeros((I * H // 256, 66), np.uint8)
    iq[:, 0:2] = [0x00, 0x1C]    # d = 2^-8
    iq[:, 2:] = rng.integers(0, 256, (iq.shape[0], 64))
    for g in range(8):
        iq[:, 2 + 8 * g + 7] &= 0x0F   # s = 0
    q2 = rng.integers(0, 256, (H * I // 256, 84)).astype(np.uint8)
    q2[:, :16] &= 0x0F               # m = 0
    q2[:, 80:82] = [0x00, 0x1C]
    q2[:, 82:84] = 0
    lay = dict(H=H, I=I, E=1, k=1, W_r=np.zeros((1, H), np.float32), b_r=None, grid=grid,
               gate=[iq], up=[iq], down=[q2], sh_gate=None, sh_up=None, sh_down=None)
    Wg = orc.dequant_iq2xxs(iq, grid)
    assert np.array_equal(orc.bf16_round(Wg), Wg)
    Wd = orc.dequant_q2k(q2)
    assert np.array_equal(orc.bf16_round(Wd), Wd)
    x = synth.tokens(2, H, seed=13, dtype=torch.bfloat16).float().numpy()
    out0, _, _ = orc.moe_forward(lay, x, mode=0)
    out1, _, _ = orc.moe_forward(lay, x, mode=1)
    # per-element bound: |sum_i Wd_ri (h_i - bf16(h_i))| <= 2^-8 sum_i |Wd_ri h_i|
    Wdm = Wd.reshape(H, I).astype(np.float64)
    Wgm = Wg.reshape(I, H).astype(np.float64)
    g = x.astype(np.float64) @ Wgm.T
    h = g / (1 + np.exp(-g)) * g
    bound = 2.0 ** -8 * (np.abs(h) @ np.abs(Wdm).T) * 1.001
    assert np.all(np.abs(out1 - out0) <= bound + 1e-30)
    assert np.abs(out1 - out0).max() > 0


def _bf16_reading_dense(Wg, Wu, Wd, x, round_w=True, round_x=True, round_h=True):
    """The bf16 tensor-core reading written with torch library routines: the
    dequantized weights, x and h rounded to bfloat16 by torch (h first to
    binary32, as a kernel holding it in an fp32 register would), sums in fp64."""
    def r(a, on):
        t = torch.from_numpy(np.asarray(a, np.float32))
        return (t.to(torch.bfloat16) if on else t).to(torch.float64)

    X = r(x, round_x)
    g = X @ r(Wg, round_w).T
    u = X @ r(Wu, round_w).T
    h = torch.nn.functional.silu(g) * u
    if round_h:
        h = h.to(torch.float32).to(torch.bfloat16).to(torch.float64)
    return (h @ r(Wd, round_w).T).numpy()


def test_bf16_reading_matches_torch_bf16_dense(orc):
    """Pin of the oracle's bf16 reading (mode 1, the prefill plan's rounding
    points: x, the dequantized routed weights and h rounded to bfloat16, sums in
    fp64) on weights and activations that bf16 does NOT represent exactly:
    one routed expert (E = k = 1, weight 1), no shared expert, against torch's
    bfloat16 conversion and fp64 matmuls.  Dropping any one of the three
    roundings moves the result far outside the 1e-12 tolerance, so a reading
    that forgot one of them fails here."""
    L = synth.float_layer(synth.Shape(H=256, I=128, E=1, k=1), 21)
    grid = L["grid"].numpy()
    gate = orc.pack_iq2xxs(L["gate_f"][0].numpy(), grid)
    up = orc.pack_iq2xxs(L["up_f"][0].numpy(), grid)
    down = orc.pack_q2k(L["down_f"][0].numpy())
    lay = dict(H=256, I=128, E=1, k=1, W_r=L["W_r"].numpy(), b_r=None, grid=grid, gate=[gate], up=[up],
               down=[down], sh_gate=None, sh_up=None, sh_down=None)
    Wg = orc.dequant_iq2xxs(gate, grid).reshape(128, 256)
    Wu = orc.dequant_iq2xxs(up, grid).reshape(128, 256)
    Wd = orc.dequant_q2k(down).reshape(256, 128)
    x = synth.tokens(3, 256, seed=22).numpy()          # binary32, not bf16-exact
    # the inputs really need rounding: most weights and x values are not bf16 numbers
    for a in (Wg, Wu, Wd, x):
        assert np.mean(orc.bf16_round(a) != a) > 0.5
    out, ids, w = orc.moe_forward(lay, x, mode=1)
    assert np.all(ids == 0) and np.all(w == 1.0)
    ref = _bf16_reading_dense(Wg, Wu, Wd, x)
    scale = np.abs(ref).max()
    assert np.abs(out - ref).max() <= 1e-12 * scale
    for miss in (dict(round_w=False), dict(round_x=False), dict(round_h=False)):
        alt = _bf16_reading_dense(Wg, Wu, Wd, x, **miss)
        assert np.abs(alt - out).max() > 1e-6 * scale, miss
