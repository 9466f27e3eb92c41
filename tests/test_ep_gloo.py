"""Expert parallelism's exchange steps on CPU: two and three gloo ranks, experts
split between them (dispatch to the experts' owners, the owners' experts, combine
back in slot order).

* plumbing: a stand-in expert (row times expert id + 1) makes every value
  checkable; each rank's output must equal, bit for bit, the same arithmetic
  done without any exchange, and every rank must receive exactly the rows
  whose experts it owns;
* layer: a tiny quantized layer (H 256, I 128, 8 experts, top-2) with the
  oracle's routing and dequantized experts on the owning ranks; the combined
  output must equal the oracle's one-process layer forward;
* a rank without tokens takes part in every collective and gets an empty
  output.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from bit_quantized_moe_softmax_b200 import dist as D
from bit_quantized_moe_softmax_b200 import ep


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_data(r, n, E, k, H):
    g = torch.Generator().manual_seed(1000 + r)
    x = torch.randn(n, H, generator=g)
    ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(n)]) if n else torch.zeros(0, k,
                                                                                                     dtype=torch.int64)
    w = torch.rand(n, k, generator=g)
    base = torch.randn(n, H, generator=g)
    return x, ids, w, base


def _plumbing(r, world, ns):
    E, k, H = 8, 2, 16
    x, ids, w, base = _rank_data(r, ns[r], E, k, H)
    owner = ep.expert_owner(E, world)
    seen = {}

    def local_fn(rows, eid):
        assert bool((owner[eid] == r).all())
        seen["rows"] = rows.shape[0]
        return rows * (eid + 1).to(rows.dtype)[:, None]

    out = ep.moe_forward_ep(x, ids, w, E, local_fn, base)
    ref = base.clone()
    for j in range(k):
        ref = torch.addcmul(ref, w[:, j:j + 1], x * (ids[:, j] + 1).to(x.dtype)[:, None])
    # rows this rank must receive: every rank's slots whose expert it owns
    expect = sum(int((owner[_rank_data(q, ns[q], E, k, H)[1]] == r).sum()) for q in range(world))
    return bool(torch.equal(out, ref)), seen.get("rows", 0) == expect, tuple(out.shape)


def _layer(r, world):
    import oracle as orc
    from bit_quantized_moe_softmax_b200 import synth
    from tests._util import oracle_layer, pack_with_oracle

    E, k, H, I = 8, 2, 256, 128
    L = synth.float_layer(synth.Shape(H=H, I=I, E=E, k=k), 7)
    L.update(pack_with_oracle(orc, L))
    lay = oracle_layer(L)
    x = synth.tokens(3 + r, H, seed=50 + r).numpy()
    rid, rw = orc.topk_softmax(orc.router_logits(x, lay["W_r"]), k)
    owner = ep.expert_owner(E, world)
    mats = {}
    for e in ep.local_experts(E, r, world):   # dequantize only the experts this rank owns
        mats[e] = (orc.dequant_iq2xxs(lay["gate"][e], lay["grid"]).reshape(I, H).astype(np.float64),
                   orc.dequant_iq2xxs(lay["up"][e], lay["grid"]).reshape(I, H).astype(np.float64),
                   orc.dequant_q2k(lay["down"][e]).reshape(H, I).astype(np.float64))

    def ffn(Wg, Wu, Wd, v):
        g, u = Wg @ v, Wu @ v
        return Wd @ (g / (1.0 + np.exp(-g)) * u)

    def local_fn(rows, eid):
        assert bool((owner[eid] == r).all())
        return torch.from_numpy(np.stack([ffn(*mats[int(e)], row) for row, e in zip(rows.numpy(), eid)]))

    bits = lambda a: a.astype(np.uint32) << 16
    sg, su, sd = (bits(lay[n]).view(np.float32).astype(np.float64).reshape(s)
                  for n, s in (("sh_gate", (I, H)), ("sh_up", (I, H)), ("sh_down", (H, I))))
    base = torch.from_numpy(np.stack([ffn(sg, su, sd, v) for v in x.astype(np.float64)]))
    out = ep.moe_forward_ep(torch.from_numpy(x.astype(np.float64)), torch.from_numpy(rid.astype(np.int64)),
                            torch.from_numpy(rw), E, local_fn, base).numpy()
    ref, ids, _ = orc.moe_forward(lay, x)
    return bool(np.array_equal(ids, rid)), float(np.abs(out - ref).max() / np.abs(ref).max())


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), LOCAL_RANK=str(rank),
                      WORLD_SIZE=str(world))
    try:
        r, _, w = D.init("gloo", timeout_s=60)
        res = {"plumbing": _plumbing(r, w, [5, 3, 6][:w]), "empty": _plumbing(r, w, [4, 0, 2][:w]),
               "layer": _layer(r, w)}
        D.barrier()
        q.put((r, res))
        D.finish()
    except Exception as e:  # report instead of hanging the parent
        import traceback

        q.put(("error", traceback.format_exc() + repr(e)))


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_gloo(world):
    """Two ranks (4 experts each) and three (3, 3 and 2 experts: uneven splits)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    assert all(g[0] != "error" for g in got), got
    for r, res in got:
        assert res["plumbing"][:2] == (True, True), (r, res)
        assert res["empty"][:2] == (True, True), (r, res)
        assert res["empty"][2][0] == [4, 0, 2][r]
        ids_ok, rel = res["layer"]
        assert ids_ok and rel < 1e-12, (r, rel)


def test_expert_owner_ranges():
    own = ep.expert_owner(10, 3)
    assert own.tolist() == [0, 0, 0, 0, 1, 1, 1, 2, 2, 2]
    assert list(ep.local_experts(10, 1, 3)) == [4, 5, 6]


def test_single_process_is_the_plain_combine():
    x, ids, w, base = _rank_data(0, 6, 8, 2, 16)
    out = ep.moe_forward_ep(x, ids, w, 8, lambda rows, e: rows * 2, base)
    ref = base.clone()
    for j in range(2):
        ref = torch.addcmul(ref, w[:, j:j + 1], x * 2)
    assert torch.equal(out, ref)
