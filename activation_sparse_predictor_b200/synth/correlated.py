"""A synthetic activation predictor correlated with the layer it predicts.

Input preparation only (like the rest of ``synth``): it builds predictor
weights P1 [r][d], P2 [d_ff][r] and the predictor bias c [d_ff]; it holds
none of the method's arithmetic (prediction, threshold, compaction and the
FFN run in the library and in the oracle).

The pages describe the predictor as a small per-layer model trained to
predict which neurons an input activates, at little accuracy cost (QbitAI
article, r-manual.ru, section "Что такое «разреженная активация»?").  No
trained weights exist here, so this stands in for one: the linear map
P2 P1 is the best rank-r approximation of the layer's first matrix W (W_gate
for ReGLU, W_up otherwise), taken before quantisation, and

    c_j = b_j + margin * || W[j] - (P2 P1)[j] ||_2 ,

so z_j = (P2 P1)[j] . xh + c_j estimates the pre-activation W[j] . xh + b_j,
shifted up by `margin` standard deviations of the part of it the low-rank
map misses (xh has unit rms, so that part has variance ||W[j] - (P2 P1)[j]||^2
over weight draws): a larger margin trades precision for recall.

The rank-r factors come from the randomized range finder with power
iterations and an SVD of the projected matrix (Halko, Martinsson and Tropp,
"Finding structure with randomness", SIAM Review 2011, algorithms 4.4 and
5.1), in float64 on the host, or float32 on a CUDA device when one is given.
P1's rows are the top right singular vectors, P2 = U_r diag(s_r).
"""
from __future__ import annotations

import math

import numpy as np

from . import T_GATE, T_UP, Workload, biases, fill_host, key


def first_matrix_unquantised(w: Workload, layer: int) -> np.ndarray:
    """The layer's first matrix [d_ff][d_model] as the generator draws it,
    before binary16 rounding or Q4_0 encoding (float32)."""
    tid = T_GATE if w.act == "reglu" else T_UP
    return fill_host(key(w.seed, layer, tid), 1.0 / math.sqrt(w.d_model),
                     (w.d_ff, w.d_model), "f32")


def truncated_svd(W, rank: int, oversample: int = 16, power_iters: int = 2, seed: int = 0):
    """(U_r, s_r, Vt_r) of a rank-`rank` approximation of W (a torch tensor)
    by the randomized range finder with `power_iters` power iterations."""
    import torch
    m, n = W.shape
    k = min(rank + oversample, min(m, n))
    g = torch.Generator(device="cpu").manual_seed(seed)
    omega = torch.randn((n, k), generator=g, dtype=W.dtype).to(W.device)
    Q, _ = torch.linalg.qr(W @ omega)
    for _ in range(power_iters):
        Z, _ = torch.linalg.qr(W.T @ Q)
        Q, _ = torch.linalg.qr(W @ Z)
    B = Q.T @ W
    Ub, s, Vt = torch.linalg.svd(B, full_matrices=False)
    U = Q @ Ub
    return U[:, :rank], s[:rank], Vt[:rank]


def correlated_predictor(w: Workload, layer: int, margin: float = 1.0, device=None,
                         power_iters: int = 2):
    """(p1, p2, p_bias) host numpy arrays for one layer: p1 [r][d] and p2
    [d_ff][r] in the workload's predictor dtype (float16 or float32), p_bias
    [d_ff] float32.  `device`: None = float64 on the host, else a torch
    device for float32 work."""
    import torch
    W = torch.from_numpy(first_matrix_unquantised(w, layer))
    if device is None:
        W = W.double()
    else:
        W = W.to(device)
    U, s, Vt = truncated_svd(W, w.rank, power_iters=power_iters, seed=w.seed * 1000 + layer)
    dt = np.float16 if w.p_dtype == "f16" else np.float32
    p1 = Vt.double().cpu().numpy().astype(dt)
    p2 = (U * s[None, :]).double().cpu().numpy().astype(dt)
    # what the stored (rounded) factors miss, row by row
    A = torch.from_numpy(p2.astype(np.float64)).to(W.device, W.dtype) @ \
        torch.from_numpy(p1.astype(np.float64)).to(W.device, W.dtype)
    resid = torch.linalg.vector_norm(W - A, dim=1)
    c = torch.from_numpy(biases(w).astype(np.float64)).to(W.device, W.dtype) + margin * resid
    return p1, p2, c.double().cpu().numpy().astype(np.float32)
