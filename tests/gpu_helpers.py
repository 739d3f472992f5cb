"""Helpers of the GPU parity tests: device layers from the seeded generator,
mask comparison with the threshold band, tolerances."""
from __future__ import annotations

import numpy as np

from activation_sparse_predictor_b200 import synth

BAND = 1e-4          # neurons whose oracle logit lies this close to the threshold are exempt
TOL = {"f32": 1e-5, "f16": 5e-3, "q4_0": 5e-3}  # relative L2 of FFN outputs


def pi_mod():
    from activation_sparse_predictor_b200 import pi
    return pi


def device_layer(w, layer: int, device="cuda", packed: bool = False):
    """(pi.Layer, raw tensors) of layer `layer`, generated in place on the GPU;
    packed=True stores each neuron's weights as one record (row strides)."""
    pi = pi_mod()
    t = synth.layer_device(w, layer, device)
    keep = {k: t[k] for k in ("w_gate", "w_up", "w_down_t", "bias", "p1", "p2", "p_bias") if k in t}
    if packed:
        return pi.Layer.packed(w, keep), t
    return pi.Layer.from_workload(w, keep), t


def unpack_bits(words: np.ndarray, n: int) -> np.ndarray:
    words = np.ascontiguousarray(words, dtype=np.uint32)
    bits = np.unpackbits(words.view(np.uint8), bitorder="little")
    return bits[:n].astype(bool), bits[n:]


def check_mask(gpu_words: np.ndarray, z_ref: np.ndarray, F: int, H: int, theta: float,
               band: float = BAND):
    """GPU mask == oracle decision outside the band; tail bits zero.
    Returns the number of (allowed) disagreements inside the band."""
    got, tail = unpack_bits(gpu_words, F)
    j = np.arange(F)
    want = (j < H) | ((j >= H) & (z_ref > theta))
    diff = got != want
    allowed = (j >= H) & (np.abs(z_ref - theta) <= band)
    bad = diff & ~allowed
    assert not bad.any(), f"mask mismatch outside the band at neurons {np.flatnonzero(bad)[:10]}"
    assert not tail.any(), "bits beyond d_ff must be 0"
    return int(diff.sum())


def words_np(t) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)
