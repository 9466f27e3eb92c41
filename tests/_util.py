"""Helpers shared by the tests: oracle-side views of synthetic layers, error metrics."""
import numpy as np
import torch


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_layer(layer: dict, experts=None) -> dict:
    import oracle

    return oracle.layer_from_torch(layer, experts)


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))


def pack_with_oracle(orc, layer: dict) -> dict:
    """Canonical blocks of a float layer packed by the oracle's packers."""
    grid = layer["grid"].numpy()
    E = layer["E"]
    gate = np.stack([orc.pack_iq2xxs(layer["gate_f"][e].numpy(), grid) for e in range(E)])
    up = np.stack([orc.pack_iq2xxs(layer["up_f"][e].numpy(), grid) for e in range(E)])
    down = np.stack([orc.pack_q2k(layer["down_f"][e].numpy()) for e in range(E)])
    return dict(gate=torch.from_numpy(gate), up=torch.from_numpy(up), down=torch.from_numpy(down))


def pack_q4_with_oracle(orc, layer: dict) -> dict:
    """Q4_K-style blocks of a float layer's three expert matrices, packed by the oracle."""
    E = layer["E"]
    out = {n: torch.from_numpy(np.stack([orc.pack_q4k(layer[n + "_f"][e].numpy()) for e in range(E)]))
           for n in ("gate", "up", "down")}
    out["expert_bits"] = 4
    return out
