"""Small shared test helpers: tiny seeded layers and float64 library decodes."""
from __future__ import annotations

import numpy as np

from activation_sparse_predictor_b200 import synth


def small_workload(act="relu", w_dtype="f32", p_dtype="f32", d=64, F=256, r=32, hot=0,
                   seed=11, mean=0.2, alpha=1.0, n_layers=1) -> synth.Workload:
    return synth.Workload(
        name=f"test_{act}_{d}x{F}_{w_dtype}", act=act, d_model=d, d_ff=F, rank=r,
        n_layers=n_layers, hot=hot, w_dtype=w_dtype, p_dtype=p_dtype, seed=seed, tau=0.5,
        p_rule=("mean", mean, alpha), steps=4)


def np_decode(a, dtype: str) -> np.ndarray:
    """float64 matrix from stored weights, using numpy's own conversions for
    f32/f16 and a vectorised Q4_0 decode (pinned separately by hand blocks)."""
    if dtype in ("f32", "f16"):
        return np.asarray(a).astype(np.float64)
    qs, sc = a
    rows, nb, _ = qs.shape
    lo = (qs & 0x0F).astype(np.int32)          # elements 0..15 of each block
    hi = (qs >> 4).astype(np.int32)            # elements 16..31
    q = np.concatenate([lo, hi], axis=2)       # [rows][nb][32]
    s = np.asarray(sc).view(np.float16).astype(np.float64)[:, :, None]
    return ((q - 8) * s).reshape(rows, nb * 32)


def torch_layer_f64(L: dict):
    """Decoded float64 torch tensors of a layer (independent of the oracle)."""
    import torch
    w = L["workload"]
    out = {}
    for k in ("w_gate", "w_up", "w_down_t"):
        if k in L:
            out[k] = torch.from_numpy(np_decode(L[k], w.w_dtype))
    for k in ("p1", "p2"):
        out[k] = torch.from_numpy(np_decode(L[k], w.p_dtype))
    out["bias"] = torch.from_numpy(np.asarray(L["bias"], np.float64))
    out["p_bias"] = torch.from_numpy(np.asarray(L["p_bias"], np.float64))
    return out


def torch_dense_ffn(L: dict, xh: np.ndarray) -> np.ndarray:
    """Dense FFN with torch float64 matmul + relu (a library special case)."""
    import torch
    T = torch_layer_f64(L)
    x = torch.from_numpy(np.asarray(xh, np.float64))
    if L["workload"].act == "relu":
        h = torch.relu(T["w_up"] @ x + T["bias"])
    elif L["workload"].act == "relu2":
        h = torch.relu(T["w_up"] @ x + T["bias"]) ** 2
    else:
        h = torch.relu(T["w_gate"] @ x + T["bias"]) * (T["w_up"] @ x)
    return (T["w_down_t"].T @ h).numpy()


def unit_rms(rng, d: int) -> np.ndarray:
    x = rng.standard_normal(d)
    return x / np.sqrt(np.mean(x * x))
