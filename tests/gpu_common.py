"""Shared helpers of the GPU parity tests: move seeded inputs to the device, run the library through its
binding, and build the oracle's reference from the same host inputs (never from a GPU result)."""

import numpy as np
import torch

from oracle import linear as L
from oracle import nf4 as O


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def dev(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        t = torch.from_numpy(t)
    return t.cuda().contiguous()


def lora_or_none(d):
    if d["r"] == 0:
        return None, None
    return dev(d["A"]), dev(d["B"])


def oracle_weight(W: np.ndarray) -> np.ndarray:
    """Wd [N,K] fp64 from the oracle's own quantization of the host weight."""
    N, K = W.shape
    codes, absmax = O.nf4_quantize(W)
    return L.dequantized_weight(codes, absmax, N, K)


def assert_close(got, ref, what: str):
    res = L.compare(f64(got), f64(ref))
    assert res["ok"], f"{what}: rel_fro={res['rel_fro']:.3e} max_abs_frac={res['max_abs_frac']:.3e}"
    return res
