"""Pins of the CPU oracle to facts outside itself.

Each pin takes an ``oracle.Oracle`` and raises AssertionError on a mismatch.
They are run against the real oracle (test_oracle_pins.py) and against
copies with planted mistakes (test_oracle_mutants.py), which must each fail
at least one pin.  What each pin rests on:

* hand-computed dyadic examples (tests/golden/*.json), exact;
* float64 library routines on tiny sizes (numpy's binary16 conversion,
  torch float64 matmul + relu), within 1e-12;
* invariants of the method: sparse == dense on the true active set
  (bitwise), hot-prefix invariance of the hot/cold split (bitwise),
  additivity over a partition of the neuron set, permutation invariance;
* brute force over every mask of 16 neurons for the compaction.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from activation_sparse_predictor_b200 import synth
from helpers import np_decode, small_workload, torch_dense_ffn, torch_layer_f64, unit_rms

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _dyadic_layer(act: str) -> dict:
    g = _golden("dyadic_ffn.json")
    f32 = lambda a: np.asarray(a, np.float32)
    L = {"meta": dict(d_model=4, d_ff=4, rank=1, hot=0, act=act, w_dtype="f32", p_dtype="f32"),
         "w_down_t": f32(g["w_down_t"]), "bias": f32(g["bias"]),
         "p1": np.zeros((1, 4), np.float32), "p2": np.zeros((4, 1), np.float32),
         "p_bias": None}
    if act in ("relu", "relu2"):
        L["w_up"] = f32(g["first_matrix"])
    else:
        L["w_gate"] = f32(g["first_matrix"])
        L["w_up"] = f32(g["reglu_up"])
    return L, g


# --------------------------------------------------------------- primitives

def pin_half_decode_all_patterns(orc):
    """binary16 decode == numpy's float16 -> float64 for every finite pattern."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    fin = np.isfinite(ref)
    got = np.array([orc.half_to_double(int(b)) for b in bits[fin][::7]])
    assert np.array_equal(got, ref[fin][::7])
    for b, v in [(0x3C00, 1.0), (0xC000, -2.0), (0x7BFF, 65504.0), (0x0001, 2.0 ** -24),
                 (0x0400, 2.0 ** -14), (0x3800, 0.5), (0x8000, -0.0)]:
        assert orc.half_to_double(b) == v


def pin_q4_0_hand_block(orc):
    """A hand-built Q4_0 block decodes to (q - 8) * s exactly."""
    # element k has code k % 16 for k < 16 and 15 - (k % 16) for k >= 16
    codes = [k % 16 for k in range(16)] + [15 - (k % 16) for k in range(16)]
    qs = np.array([[[codes[k] | (codes[k + 16] << 4) for k in range(16)]]], np.uint8)
    sc = np.array([[0x3800]], np.uint16)  # 0.5
    got = orc.decode_matrix((qs, sc), "q4_0", 32)[0]
    want = [(c - 8) * 0.5 for c in codes]
    assert list(got) == want, (list(got), want)
    # a second block with a negative scale: -0.25 = 0xB400
    sc2 = np.array([[0xB400]], np.uint16)
    got2 = orc.decode_matrix((qs, sc2), "q4_0", 32)[0]
    assert list(got2) == [(c - 8) * -0.25 for c in codes]


def pin_q4_0_matches_numpy_decode(orc):
    """Oracle Q4_0 decode == the vectorised numpy decode on generated blocks."""
    k = synth.key(7, 0, 0)
    qs, sc = synth.fill_host(k, 0.05, (3, 128), "q4_0")
    got = orc.decode_matrix((qs, sc), "q4_0", 128)
    assert np.array_equal(got, np_decode((qs, sc), "q4_0"))


def pin_rmsnorm_closed_form(orc):
    """x = (3, 4, 0, 0): mean square 6.25, so xh = (1.2, 1.6, 0, 0)/sqrt(1 + 1.6e-7)."""
    got = orc.rmsnorm(np.array([3, 4, 0, 0], np.float32))
    f = 1.0 / math.sqrt(1.0 + 1.6e-7)
    assert np.allclose(got, [1.2 * f, 1.6 * f, 0, 0], rtol=1e-13, atol=0)
    # constant vector c: every entry c / sqrt(c^2 + 1e-6)
    got = orc.rmsnorm(np.full(8, 0.5, np.float32))
    assert np.allclose(got, 0.5 / math.sqrt(0.25 + 1e-6), rtol=1e-14)


# ---------------------------------------------------------------------- FFN

def pin_dyadic_ffn(orc):
    """Hand-computed ReLU, ReGLU and squared ReLU layers: h and y exact."""
    for act in ("relu", "reglu", "relu2"):
        L, g = _dyadic_layer(act)
        h, y = orc.ffn(L, np.array(g["xh"]), np.ones(4, np.uint8))
        assert list(h) == g[f"{act}_h"], (act, list(h))
        assert list(y) == g[f"{act}_y"], (act, list(y))


def pin_dense_vs_torch_f64(orc):
    """Dense FFN == torch float64 matmul + relu (squared for squared ReLU),
    tiny sizes, all weight dtypes."""
    rng = np.random.default_rng(3)
    for act in ("relu", "reglu", "relu2"):
        for wdt in ("f32", "f16", "q4_0"):
            w = small_workload(act, wdt, d=64, F=96, r=16, seed=21)
            L = synth.layer_host(w, 0)
            xh = unit_rms(rng, w.d_model)
            y = orc.dense_ffn(L, xh)
            ref = torch_dense_ffn(L, xh)
            assert np.allclose(y, ref, rtol=1e-12, atol=1e-13), (act, wdt)


def _true_set(orc, L, xh):
    h, _ = orc.ffn(L, xh, np.ones(L["workload"].d_ff, np.uint8))
    return h != 0.0


def pin_sparse_true_mask_equals_dense(orc):
    """With S = {j : activation > 0}, sparse == dense bitwise."""
    rng = np.random.default_rng(4)
    for act in ("relu", "reglu", "relu2"):
        w = small_workload(act, "f16", d=64, F=256, r=16, seed=22)
        L = synth.layer_host(w, 0)
        xh = unit_rms(rng, w.d_model)
        dense = orc.dense_ffn(L, xh)
        T = _true_set(orc, L, xh)
        assert 0 < T.sum() < w.d_ff
        _, ys = orc.ffn(L, xh, T.astype(np.uint8))
        assert np.array_equal(ys, dense)
        # the same through the list + hot-prefix path
        ys2 = orc.sparse_ffn(L, xh, np.flatnonzero(T).astype(np.int32), hot=0)
        assert np.array_equal(ys2, dense)


def pin_all_ones_mask_equals_dense(orc):
    """All neurons listed, no hot prefix: sparse == dense bitwise."""
    rng = np.random.default_rng(5)
    w = small_workload("reglu", "q4_0", d=64, F=128, r=16, seed=23)
    L = synth.layer_host(w, 0)
    xh = unit_rms(rng, w.d_model)
    ys = orc.sparse_ffn(L, xh, np.arange(w.d_ff, dtype=np.int32), hot=0)
    assert np.array_equal(ys, orc.dense_ffn(L, xh))


def pin_hot_prefix_invariance(orc):
    """Hot/cold split does not change the result: hot=H with list idx equals
    hot=0 with list [0,H) U idx, bitwise (the neurons 3,4,5 example)."""
    rng = np.random.default_rng(6)
    w = small_workload("relu", "f16", d=64, F=256, r=16, hot=64, seed=24)
    L = synth.layer_host(w, 0)
    L["bias"] = np.full(w.d_ff, 4.0, np.float32)  # every neuron active: each one counts
    xh = unit_rms(rng, w.d_model)
    idx = np.sort(rng.choice(np.arange(64, 256), 40, replace=False)).astype(np.int32)
    a = orc.sparse_ffn(L, xh, idx, hot=64)
    b = orc.sparse_ffn(L, xh, np.concatenate([np.arange(64), idx]).astype(np.int32), hot=0)
    assert np.array_equal(a, b)
    # the neuron set itself is [0, H) U idx
    want = np.zeros(w.d_ff, np.uint8)
    want[:64] = 1
    want[idx] = 1
    assert np.array_equal(orc.rowset(w.d_ff, 64, idx), want)
    # and differs from the set without the hot prefix
    assert not np.array_equal(a, orc.sparse_ffn(L, xh, idx, hot=0))


def pin_partition_additivity(orc):
    """y(S1 U S2) = y(S1) + y(S2) for disjoint S1, S2 (merge of partial sums)."""
    rng = np.random.default_rng(7)
    for act in ("relu", "reglu", "relu2"):
        w = small_workload(act, "f32", d=64, F=200, r=16, seed=25)
        L = synth.layer_host(w, 0)
        xh = unit_rms(rng, w.d_model)
        part = rng.integers(0, 3, w.d_ff)
        s1 = (part == 1).astype(np.uint8)
        s2 = (part == 2).astype(np.uint8)
        _, y1 = orc.ffn(L, xh, s1)
        _, y2 = orc.ffn(L, xh, s2)
        _, y12 = orc.ffn(L, xh, s1 | s2)
        assert np.allclose(y12, y1 + y2, rtol=1e-12, atol=1e-14)
        assert np.abs(y1).sum() > 0 and np.abs(y2).sum() > 0


def pin_permutation_invariance(orc):
    """Permuting neurons (rows of all matrices and the bias) leaves y unchanged."""
    rng = np.random.default_rng(8)
    w = small_workload("reglu", "f32", d=64, F=160, r=16, seed=26)
    L = synth.layer_host(w, 0)
    xh = unit_rms(rng, w.d_model)
    perm = rng.permutation(w.d_ff)
    P = dict(L)
    for k in ("w_gate", "w_up", "w_down_t", "bias"):
        P[k] = np.ascontiguousarray(L[k][perm])
    y = orc.dense_ffn(L, xh)
    yp = orc.dense_ffn(P, xh)
    assert np.allclose(yp, y, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- predictor

def pin_dyadic_predictor(orc):
    """Hand-computed predictor: u, z, masks and lists exact."""
    g = _golden("dyadic_predictor.json")
    L = {"meta": dict(d_model=2, d_ff=4, rank=2, hot=1, act="relu", w_dtype="f32",
                      p_dtype="f32"),
         "w_up": np.zeros((4, 2), np.float32), "w_down_t": np.zeros((4, 2), np.float32),
         "bias": None, "p1": np.asarray(g["p1"], np.float32),
         "p2": np.asarray(g["p2"], np.float32), "p_bias": np.asarray(g["p_bias"], np.float32)}
    u, z = orc.predict(L, np.array(g["xh"]))
    assert list(u) == g["u"]
    assert list(z[1:]) == g["z_cold"]
    for tau, key in ((0.5, "0_5"), (0.75, "0_75")):
        theta = float(np.float32(math.log(tau / (1 - tau))))
        m = orc.mask(z, 4, 1, theta)
        assert int(m[0]) == g[f"mask_tau_{key}"], (tau, int(m[0]))
        assert list(orc.compact(m, 4, 1)) == g[f"list_tau_{key}"]


def pin_predictor_vs_torch_f64(orc):
    """z = P2 (P1 xh) + c for cold neurons, against torch float64."""
    import torch
    rng = np.random.default_rng(9)
    for pdt in ("f32", "f16"):
        w = small_workload("relu", "f32", pdt, d=64, F=192, r=24, hot=32, seed=27)
        L = synth.layer_host(w, 0)
        xh = unit_rms(rng, w.d_model)
        u, z = orc.predict(L, xh)
        T = torch_layer_f64(L)
        x = torch.from_numpy(xh)
        uref = (T["p1"] @ x)
        zref = (T["p2"] @ uref + T["p_bias"]).numpy()
        assert np.allclose(u, uref.numpy(), rtol=1e-12, atol=1e-13)
        assert np.allclose(z[32:], zref[32:], rtol=1e-12, atol=1e-13)
        assert np.all(np.isinf(z[:32]))


def pin_threshold_is_sigmoid_test(orc):
    """Away from the 1e-4 band, (z > logit(tau)) == (sigmoid(z) > tau)."""
    rng = np.random.default_rng(10)
    F, H = 512, 0
    z = rng.standard_normal(F) * 3
    for tau in (0.2, 0.5, 0.9):
        theta = float(np.float32(math.log(tau / (1 - tau))))
        m = orc.mask(z, F, H, theta)
        bits = (m[np.arange(F) // 32] >> (np.arange(F) % 32).astype(np.uint32)) & 1
        sig = 1.0 / (1.0 + np.exp(-z))
        away = np.abs(z - theta) > 1e-4
        assert np.array_equal(bits[away].astype(bool), (sig > tau)[away])


def pin_mask_hot_bits_and_tail(orc):
    """Hot neurons always set; bits beyond d_ff zero."""
    F, H = 70, 33
    z = np.full(F, -5.0)
    m = orc.mask(z, F, H, 0.0)
    assert int(m[0]) == 0xFFFFFFFF and int(m[1]) == 1 and int(m[2]) == 0


# ------------------------------------------------------------- compaction

def pin_compaction_bruteforce_16(orc):
    """Every mask of 16 neurons, begin in {0, 5}: the ascending set-bit list."""
    for mword in range(1 << 16):
        m = np.array([mword], np.uint32)
        for begin in (0, 5):
            got = orc.compact(m, 16, begin)
            want = [j for j in range(begin, 16) if (mword >> j) & 1]
            if list(got) != want:
                raise AssertionError((mword, begin, list(got), want))


def pin_compaction_union_and_large(orc):
    """Union = OR of token masks; a large random mask equals numpy's nonzero."""
    rng = np.random.default_rng(12)
    F = 49152
    words = F // 32
    masks = rng.integers(0, 2 ** 32, (4, words), dtype=np.uint64).astype(np.uint32)
    masks &= rng.integers(0, 2 ** 32, (4, words), dtype=np.uint64).astype(np.uint32)
    bits = np.unpackbits(masks.view(np.uint8), bitorder="little").reshape(4, F)
    for begin in (0, 9728):
        got = orc.compact(masks, F, begin)
        want = np.flatnonzero(bits.any(axis=0))
        assert np.array_equal(got, want[want >= begin])
        got1 = orc.compact(masks[2], F, begin)
        want1 = np.flatnonzero(bits[2])
        assert np.array_equal(got1, want1[want1 >= begin])


# ------------------------------------------------------------------ stack

def pin_layer_forward_residual(orc):
    """With W_down = 0 the layer is the identity on x; otherwise x + y of the
    predicted set."""
    rng = np.random.default_rng(13)
    w = small_workload("relu", "f32", d=64, F=128, r=16, hot=32, seed=28)
    L = synth.layer_host(w, 0)
    x = rng.standard_normal(64).astype(np.float32) * 3
    Z = dict(L)
    Z["w_down_t"] = np.zeros_like(L["w_down_t"])
    xo, m, z = orc.layer_forward(Z, x, 0.5)
    assert np.array_equal(xo, x.astype(np.float64))
    xo, m, z = orc.layer_forward(L, x, 0.5)
    xh = orc.rmsnorm(x)
    idx = orc.compact(m, 128, 32)
    y = orc.sparse_ffn(L, xh, idx, hot=32)
    assert np.array_equal(xo, x.astype(np.float64) + y)
    assert np.abs(y).sum() > 0


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
