"""The seeded input generator: rounding, distribution, Q4_0 encoding and the
calibration of firing probabilities.  CPU only (host/device bit equality is
checked in the GPU tests)."""
import math

import numpy as np
import pytest

from activation_sparse_predictor_b200 import synth
from helpers import np_decode, small_workload


def test_half_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 5, 20000),
        # exact ties between neighbouring binary16 values
        (np.arange(1, 2000) + 0.5) * 2.0 ** -10,
        (np.arange(1, 2000) + 0.5) * 2.0 ** -24,
        np.array([65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -25, 2.0 ** -26, 3 * 2.0 ** -26]),
    ])
    v = np.concatenate([v, -v])
    got = np.array([synth.half_bits(x) for x in v], np.uint16)
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


def test_gauss_moments_and_determinism():
    k = synth.key(1, 2, 3)
    x = synth.fill_host(k, 1.0, (200000,), "f64")
    assert abs(x.mean()) < 0.01
    assert abs(x.var() - 1.0) < 0.01
    assert abs(np.mean(x ** 4) - 3.0) < 0.1   # Irwin-Hall(12) kurtosis 2.9
    assert np.array_equal(x, synth.fill_host(k, 1.0, (200000,), "f64"))
    assert synth.gauss(k, 17) == x[17]
    assert synth.key(1, 2, 3) != synth.key(1, 2, 4) != synth.key(2, 2, 3)


def test_f16_f32_are_rounded_f64():
    k = synth.key(5, 0, 1)
    x = synth.fill_host(k, 0.1, (4096,), "f64")
    assert np.array_equal(synth.fill_host(k, 0.1, (4096,), "f32"), x.astype(np.float32))
    assert np.array_equal(synth.fill_host(k, 0.1, (4096,), "f16").view(np.uint16),
                          x.astype(np.float16).view(np.uint16))


def test_q4_0_encoder_round_trip():
    k = synth.key(6, 0, 0)
    rows, cols, sigma = 64, 256, 1 / math.sqrt(256)
    raw = synth.fill_host(k, sigma, (rows, cols), "f64")
    qs, sc = synth.fill_host(k, sigma, (rows, cols), "q4_0")
    dec = np_decode((qs, sc), "q4_0")
    s = np.repeat(np.abs(sc.view(np.float16).astype(np.float64)), 32, axis=1)
    q = np.concatenate([qs & 15, qs >> 4], axis=2).reshape(rows, cols)
    err = np.abs(raw - dec)
    unclamped = q != 15
    assert np.all(err[unclamped] <= s[unclamped] / 2 * (1 + 1e-12))
    assert np.all(err <= s * (1 + 1e-12))
    # the largest-magnitude element of every block encodes to q = 0
    blocks = raw.reshape(rows, cols // 32, 32)
    imax = np.argmax(np.abs(blocks), axis=2)
    qb = q.reshape(rows, cols // 32, 32)
    assert np.all(np.take_along_axis(qb, imax[..., None], axis=2) == 0)


def test_q4_0_zero_block():
    qs, sc = synth.fill_host(synth.key(0, 0, 0), 0.0, (2, 64), "q4_0")
    assert np.all(qs == 0x88)
    assert np.all(sc.view(np.float16).astype(np.float64) == 0.0)


@pytest.mark.parametrize("name,hot,mean,top20", [
    ("relullama7b_reglu_4096x11008_f16", 2176, 0.12, 0.65),
    ("falcon40b_relu_8192x32768_f16", 6528, 0.08, 0.75),
    ("llama2_70b_reglu_8192x28672_q4_0", 5632, 0.15, 0.62),
    ("opt175b_relu_12288x49152_f16", 9728, 0.05, 0.76),
])
def test_power_law_profiles(name, hot, mean, top20):
    w = synth.WORKLOADS[name]
    p = synth.activation_probs(w)
    assert w.hot == hot
    assert abs(p.mean() - mean) < 1e-9
    assert p.max() == 0.95 and np.all(np.diff(p) <= 0)
    mass = p[: int(0.2 * w.d_ff)].sum() / p.sum()
    assert abs(mass - top20) < 0.01, mass


def test_tiny_profile_is_explicit():
    w = synth.WORKLOADS["tiny_relu_512x2048_f32"]
    p = synth.activation_probs(w)
    j = np.arange(1, 2049)
    assert np.array_equal(p, np.minimum(0.95, 0.5 * j ** -0.6))
    assert w.hot == 0 and w.d_ff == 2048 and w.rank == 64
    b = synth.biases(w)
    assert b[0] == 0.0  # p_0 = 0.5


def test_firing_calibration():
    """Over random unit-rms inputs neuron j fires with probability
    Phi(b_j / ||W_j||), and the mean density is near the target."""
    from scipy.special import ndtr
    w = small_workload("relu", "f32", d=512, F=256, r=16, seed=31, mean=0.15, alpha=1.0)
    L = synth.layer_host(w, 0)
    rng = np.random.default_rng(1)
    n = 4096
    X = rng.standard_normal((n, 512))
    X /= np.sqrt((X * X).mean(axis=1, keepdims=True))
    W = L["w_up"].astype(np.float64)
    b = L["bias"].astype(np.float64)
    fire = ((X @ W.T + b) > 0).mean(axis=0)
    p_exp = ndtr(b / np.linalg.norm(W, axis=1))
    sd = np.sqrt(p_exp * (1 - p_exp) / n)
    assert np.all(np.abs(fire - p_exp) <= 4 * sd + 1e-3)
    assert abs(fire.mean() - 0.15) < 0.02
    # the predictor is calibrated the same way through P2 P1
    P = L["p2"].astype(np.float64) @ L["p1"].astype(np.float64)
    pred = ((X @ P.T + L["p_bias"]) > 0).mean(axis=0)
    assert abs(pred.mean() - 0.15) < 0.03


def test_threshold_logit():
    assert synth.threshold_logit(0.5) == 0.0
    assert synth.threshold_logit(0.75) == float(np.float32(math.log(3.0)))
