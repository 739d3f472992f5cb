"""Pins of the correlated synthetic predictor (input preparation): its rank-r
map against numpy's exact SVD, its near-optimal error at the default
settings, and the bias calibration against numpy row norms."""
import numpy as np
import pytest

from activation_sparse_predictor_b200 import synth
from activation_sparse_predictor_b200.synth import correlated as C

torch = pytest.importorskip("torch")


def _w(act="reglu", d=64, F=96, r=16, pdt="f32", seed=5):
    return synth.Workload("corr_test", act, d, F, r, 1, 0, "f16", pdt, seed=seed, tau=0.5,
                          p_rule=("mean", 0.2, 1.0), steps=1)


def test_full_sketch_equals_exact_truncated_svd():
    """With the sketch as wide as the matrix, the factors give numpy's exact
    rank-r truncation (Eckart-Young)."""
    w = _w()
    W = C.first_matrix_unquantised(w, 0).astype(np.float64)
    U, s, Vt = np.linalg.svd(W, full_matrices=False)
    Wr = (U[:, :16] * s[:16]) @ Vt[:16]
    Ur, sr, Vtr = C.truncated_svd(torch.from_numpy(W), 16, oversample=64, power_iters=2)
    A = ((Ur * sr[None, :]) @ Vtr).numpy()
    assert np.linalg.norm(A - Wr) / np.linalg.norm(Wr) < 1e-10
    assert np.allclose(sr.numpy(), s[:16], rtol=1e-10)
    # orthonormal right factors
    assert np.allclose(Vtr.numpy() @ Vtr.numpy().T, np.eye(16), atol=1e-10)


def test_default_sketch_is_near_optimal():
    """Default sketch: Frobenius error within 3 % of the optimal rank-r error."""
    w = _w(d=512, F=1500, r=64)
    W = C.first_matrix_unquantised(w, 0).astype(np.float64)
    s = np.linalg.svd(W, compute_uv=False)
    opt = np.sqrt((s[64:] ** 2).sum())
    Ur, sr, Vtr = C.truncated_svd(torch.from_numpy(W), 64)
    err = np.linalg.norm(W - ((Ur * sr[None, :]) @ Vtr).numpy())
    assert opt <= err <= 1.03 * opt


@pytest.mark.parametrize("act,pdt", [("reglu", "f32"), ("relu", "f16"), ("relu2", "f32")])
def test_predictor_weights_and_bias(act, pdt):
    """p2 @ p1 is the truncation of the right matrix (gate for ReGLU, up
    otherwise), rounded to the predictor dtype; c = b + margin * row norm of
    what the truncation misses."""
    w = _w(act=act, pdt=pdt, d=128, F=200, r=32)
    p1, p2, c = C.correlated_predictor(w, 0, margin=0.75)
    assert p1.shape == (32, 128) and p2.shape == (200, 32) and c.shape == (200,)
    assert p1.dtype == (np.float16 if pdt == "f16" else np.float32) == p2.dtype
    tid = synth.T_GATE if act == "reglu" else synth.T_UP
    W = synth.fill_host(synth.key(w.seed, 0, tid), 1 / np.sqrt(128), (200, 128), "f32")
    assert np.array_equal(W, C.first_matrix_unquantised(w, 0))
    W = W.astype(np.float64)
    A = p2.astype(np.float64) @ p1.astype(np.float64)
    s = np.linalg.svd(W, compute_uv=False)
    opt = np.sqrt((s[32:] ** 2).sum())
    tol = 1.05 if pdt == "f32" else 1.10  # binary16 rounding of the factors
    assert np.linalg.norm(W - A) <= tol * opt
    resid = np.linalg.norm(W - A, axis=1)
    b = synth.biases(w).astype(np.float64)
    want = b + 0.75 * resid
    assert np.allclose(c, want, rtol=0, atol=1e-5)
    # margin 0 is the plain low-rank estimate of the pre-activation
    _, _, c0 = C.correlated_predictor(w, 0, margin=0.0)
    assert np.allclose(c0, b, atol=1e-6)
