"""Seeded synthetic workloads for the predictor-gated sparse FFN.

This module prepares inputs only: layer weights, biases, predictor weights
and input vectors, on the host (numpy) or in place on a CUDA device, with
identical bits on both sides (see ``rng.h``).  It holds none of the method's
arithmetic and is the one module that both the CPU oracle's tests and the
CUDA path's tests and benchmark use.

Workload recipe (shapes from the PowerInfer write-ups' model families:
ReluLLaMA-7B, Falcon(ReLU)-40B, Llama2-70B, OPT-175B; QbitAI article
(r-manual.ru) §"Скорость вывода до 11 раз" and §"Локальность вывода,
вызванная редкой активацией"):

* neurons are stored hot-first, so neuron j fires with probability
  p_j = min(0.95, C * (j+1)^-alpha), a power law whose constant C is
  bisected so that mean_j p_j hits the stated density (the tiny workload
  states p_j = min(0.95, 0.5 * (j+1)^-0.6) directly);
* W_gate, W_up ~ N(0, 1/d), W_down ~ N(0, 1/d_ff) (variance 1/fan_in),
  P1 ~ N(0, 1/d), P2 ~ N(0, 1/rank);
* the activation bias b_j and the predictor bias c_j are both
  Phi^-1(p_j): with a unit-rms input, W[j].x is ~N(0,1) over the weight
  draw, so neuron j fires (and is predicted) with probability p_j;
* inputs x ~ N(0, 1);
* the hot prefix is the first H = floor(0.2 d_ff / 128) * 128 neurons
  (none for the tiny workload).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libpi_synth_host.so")
DEV_LIB = os.path.join(_HERE, "libpi_synth_dev.so")

# tensor ids inside a layer's key space
T_GATE, T_UP, T_DOWN, T_P1, T_P2, T_X = 0, 1, 2, 3, 4, 5
X_LAYER_BASE = 1_000_000  # key-space "layer" of the input of decode step s


@dataclass(frozen=True)
class Workload:
    name: str
    act: str            # "relu" | "reglu" | "relu2" (squared ReLU)
    d_model: int
    d_ff: int
    rank: int
    n_layers: int
    hot: int
    w_dtype: str        # "f32" | "f16" | "q4_0"
    p_dtype: str        # "f32" | "f16"
    seed: int
    tau: float
    p_rule: tuple       # ("explicit", c, alpha) or ("mean", target, alpha)
    steps: int
    batches: tuple = (1,)
    union_batches: tuple = ()
    description: str = ""

    @property
    def nm(self) -> int:
        """Weight matrices per layer (ReLU: up, down; ReGLU: gate, up, down)."""
        return 3 if self.act == "reglu" else 2

    def scaled(self, n_layers: int) -> "Workload":
        """The same layer shape with a different number of layers."""
        kw = dict(self.__dict__)
        kw["n_layers"] = n_layers
        return Workload(**kw)


def _hot(d_ff: int) -> int:
    return (int(0.2 * d_ff) // 128) * 128


WORKLOADS = {
    "tiny_relu_512x2048_f32": Workload(
        "tiny_relu_512x2048_f32", "relu", 512, 2048, 64, 1, 0, "f32", "f32",
        seed=0, tau=0.5, p_rule=("explicit", 0.5, 0.6), steps=16,
        description="tiny ReLU FFN, 1 layer, fp32, batch 1, 16 input vectors"),
    "relullama7b_reglu_4096x11008_f16": Workload(
        "relullama7b_reglu_4096x11008_f16", "reglu", 4096, 11008, 1024, 32, _hot(11008),
        "f16", "f16", seed=2, tau=0.5, p_rule=("mean", 0.12, 1.0), steps=256,
        description="ReluLLaMA-7B-shaped ReGLU stack, 32 layers, fp16, batch 1 decode"),
    "falcon40b_relu_8192x32768_f16": Workload(
        "falcon40b_relu_8192x32768_f16", "relu", 8192, 32768, 1024, 60, _hot(32768),
        "f16", "f16", seed=3, tau=0.5, p_rule=("mean", 0.08, 1.2), steps=64,
        union_batches=(64,),
        description="Falcon-40B-shaped ReLU stack, 60 layers, fp16, batch 1 decode "
                    "and 64-token union-mask prefill"),
    "llama2_70b_reglu_8192x28672_q4_0": Workload(
        "llama2_70b_reglu_8192x28672_q4_0", "reglu", 8192, 28672, 1024, 80, _hot(28672),
        "q4_0", "f16", seed=4, tau=0.5, p_rule=("mean", 0.15, 1.0), steps=64,
        description="Llama2-70B-shaped ReGLU stack, 80 layers, Q4_0 weights, fp16 "
                    "predictor, batch 1 decode"),
    "prosparse13b_reglu_5120x13824_f16": Workload(
        "prosparse13b_reglu_5120x13824_f16", "reglu", 5120, 13824, 1024, 40, _hot(13824),
        "f16", "f16", seed=6, tau=0.5, p_rule=("mean", 0.10, 1.0), steps=64,
        description="ProSparse-Llama2-13B-shaped ReGLU stack, 40 layers, fp16, ~90% "
                    "sparse, batch 1 decode"),
    "bamboo7b_relu2_4096x14336_f16": Workload(
        "bamboo7b_relu2_4096x14336_f16", "relu2", 4096, 14336, 1024, 32, _hot(14336),
        "f16", "f16", seed=7, tau=0.5, p_rule=("mean", 0.10, 1.0), steps=64,
        description="Bamboo-7B-shaped squared-ReLU stack, 32 layers, fp16, ~90% sparse, "
                    "batch 1 decode"),
    "opt175b_relu_12288x49152_f16": Workload(
        "opt175b_relu_12288x49152_f16", "relu", 12288, 49152, 1024, 12, _hot(49152),
        "f16", "f16", seed=5, tau=0.5, p_rule=("mean", 0.05, 1.1), steps=16,
        batches=(1, 4, 16), union_batches=(64,),
        description="OPT-175B-shaped ReLU stack, 12 layers, fp16, batch 1/4/16 "
                    "per-token masks and 64 union mask"),
}
WORKLOAD_ORDER = list(WORKLOADS)


def activation_probs(w: Workload) -> np.ndarray:
    """Per-neuron firing probability p_j (float64, length d_ff)."""
    kind, a, alpha = w.p_rule
    j1 = np.arange(1, w.d_ff + 1, dtype=np.float64)
    if kind == "explicit":
        return np.minimum(0.95, a * j1 ** (-alpha))
    target = a
    lo, hi = 0.0, 1.0
    while np.minimum(0.95, hi * j1 ** (-alpha)).mean() < target:
        hi *= 2.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if np.minimum(0.95, mid * j1 ** (-alpha)).mean() < target:
            lo = mid
        else:
            hi = mid
    return np.minimum(0.95, hi * j1 ** (-alpha))


def _ndtri(p: np.ndarray) -> np.ndarray:
    from scipy.special import ndtri
    return ndtri(p)


def biases(w: Workload) -> np.ndarray:
    """b_j = c_j = Phi^-1(p_j), float32."""
    return _ndtri(activation_probs(w)).astype(np.float32)


def threshold_logit(tau: float) -> float:
    """logit(tau) computed in double, rounded to float32 (as the boundary does)."""
    return float(np.float32(math.log(tau / (1.0 - tau))))


# ----------------------------------------------------------------- host side

_host = None


def _host_lib():
    global _host
    if _host is None:
        if not os.path.exists(HOST_LIB):
            raise RuntimeError(f"synthetic-input host library missing: {HOST_LIB} "
                               "(run __graft_entry__.build())")
        lib = ctypes.CDLL(HOST_LIB)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.sy_key_of.restype = u64
        lib.sy_key_of.argtypes = [u64, u64, u64]
        lib.sy_gauss_of.restype = dbl
        lib.sy_gauss_of.argtypes = [u64, u64]
        lib.sy_half_bits_of.restype = ctypes.c_uint16
        lib.sy_half_bits_of.argtypes = [dbl]
        lib.sy_fill_f32.argtypes = [u64, dbl, i64, vp]
        lib.sy_fill_f16.argtypes = [u64, dbl, i64, vp]
        lib.sy_fill_f64.argtypes = [u64, dbl, i64, vp]
        lib.sy_fill_q4_0.argtypes = [u64, dbl, i64, i64, vp, vp]
        _host = lib
    return _host


def key(seed: int, layer: int, tensor: int) -> int:
    return int(_host_lib().sy_key_of(seed, layer, tensor))


def half_bits(v: float) -> int:
    return int(_host_lib().sy_half_bits_of(float(v)))


def gauss(k: int, e: int) -> float:
    return float(_host_lib().sy_gauss_of(k, e))


def fill_host(k: int, sigma: float, shape, dtype: str):
    """Host tensor of `shape` in dtype f64/f32/f16 (returned as float16 view)
    or q4_0 (returned as (qs uint8 [rows][cols/32][16], scales uint16 [rows][cols/32]))."""
    lib = _host_lib()
    n = int(np.prod(shape))
    if dtype == "f64":
        out = np.empty(shape, np.float64)
        lib.sy_fill_f64(k, sigma, n, out.ctypes.data)
        return out
    if dtype == "f32":
        out = np.empty(shape, np.float32)
        lib.sy_fill_f32(k, sigma, n, out.ctypes.data)
        return out
    if dtype == "f16":
        out = np.empty(shape, np.uint16)
        lib.sy_fill_f16(k, sigma, n, out.ctypes.data)
        return out.view(np.float16)
    if dtype == "q4_0":
        rows, cols = shape
        assert cols % 32 == 0
        qs = np.empty((rows, cols // 32, 16), np.uint8)
        sc = np.empty((rows, cols // 32), np.uint16)
        lib.sy_fill_q4_0(k, sigma, rows, cols, qs.ctypes.data, sc.ctypes.data)
        return qs, sc
    raise ValueError(dtype)


def _tensor_specs(w: Workload):
    """(name, tensor id, shape, sigma, dtype) of one layer's weights."""
    d, F, r = w.d_model, w.d_ff, w.rank
    specs = []
    if w.act == "reglu":
        specs.append(("w_gate", T_GATE, (F, d), 1.0 / math.sqrt(d), w.w_dtype))
    specs.append(("w_up", T_UP, (F, d), 1.0 / math.sqrt(d), w.w_dtype))
    specs.append(("w_down_t", T_DOWN, (F, d), 1.0 / math.sqrt(F), w.w_dtype))
    specs.append(("p1", T_P1, (r, d), 1.0 / math.sqrt(d), w.p_dtype))
    specs.append(("p2", T_P2, (F, r), 1.0 / math.sqrt(r), w.p_dtype))
    return specs


def layer_host(w: Workload, layer: int) -> dict:
    """One layer's tensors as host numpy arrays.

    Keys: w_gate (ReGLU only), w_up, w_down_t, p1, p2 (float32 / float16
    arrays, or for q4_0 weights a (qs, scales) pair), bias, p_bias (float32).
    """
    out = {"workload": w, "layer": layer}
    for name, tid, shape, sigma, dt in _tensor_specs(w):
        out[name] = fill_host(key(w.seed, layer, tid), sigma, shape, dt)
    b = biases(w)
    out["bias"] = b.copy()
    out["p_bias"] = b.copy()
    return out


def x_host(w: Workload, step: int, batch: int) -> np.ndarray:
    """Input vectors of decode step `step`: float32 [batch][d_model], ~N(0,1)."""
    return fill_host(key(w.seed, X_LAYER_BASE + step, T_X), 1.0, (batch, w.d_model), "f32")


# --------------------------------------------------------------- device side

_dev = None


def _dev_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(DEV_LIB):
            raise RuntimeError(f"synthetic-input device library missing: {DEV_LIB} "
                               "(run __graft_entry__.build())")
        lib = ctypes.CDLL(DEV_LIB)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.sy_dev_fill_f32.argtypes = [u64, dbl, i64, vp, vp]
        lib.sy_dev_fill_f16.argtypes = [u64, dbl, i64, vp, vp]
        lib.sy_dev_fill_q4_0.argtypes = [u64, dbl, i64, i64, vp, vp, vp]
        for f in (lib.sy_dev_fill_f32, lib.sy_dev_fill_f16, lib.sy_dev_fill_q4_0):
            f.restype = ctypes.c_int
        _dev = lib
    return _dev


def fill_device(k: int, sigma: float, shape, dtype: str, device, stream=None):
    """Device counterpart of fill_host (same bits), returning torch tensors."""
    import torch
    lib = _dev_lib()
    s = stream if stream is not None else torch.cuda.current_stream(device).cuda_stream
    n = int(np.prod(shape))
    if dtype == "f32":
        t = torch.empty(shape, dtype=torch.float32, device=device)
        rc = lib.sy_dev_fill_f32(k, sigma, n, t.data_ptr(), s)
    elif dtype == "f16":
        t = torch.empty(shape, dtype=torch.float16, device=device)
        rc = lib.sy_dev_fill_f16(k, sigma, n, t.data_ptr(), s)
    elif dtype == "q4_0":
        rows, cols = shape
        qs = torch.empty((rows, cols // 32, 16), dtype=torch.uint8, device=device)
        sc = torch.empty((rows, cols // 32), dtype=torch.float16, device=device)
        rc = lib.sy_dev_fill_q4_0(k, sigma, rows, cols, qs.data_ptr(), sc.data_ptr(), s)
        t = (qs, sc)
    else:
        raise ValueError(dtype)
    if rc != 0:
        raise RuntimeError(f"device generator launch failed: cuda error {rc}")
    return t


def layer_device(w: Workload, layer: int, device="cuda") -> dict:
    """One layer's tensors generated in place on `device` (torch tensors)."""
    import torch
    out = {"workload": w, "layer": layer}
    for name, tid, shape, sigma, dt in _tensor_specs(w):
        out[name] = fill_device(key(w.seed, layer, tid), sigma, shape, dt, device)
    b = torch.from_numpy(biases(w)).to(device)
    out["bias"] = b
    out["p_bias"] = b.clone()
    return out


def x_device(w: Workload, step: int, batch: int, device="cuda"):
    return fill_device(key(w.seed, X_LAYER_BASE + step, T_X), 1.0, (batch, w.d_model),
                       "f32", device)


def layer_nbytes(w: Workload) -> int:
    """Device bytes of one layer's weights (FFN + predictor), for sizing."""
    wb = {"f32": 4.0, "f16": 2.0, "q4_0": 18.0 / 32.0}
    ffn = w.nm * w.d_ff * w.d_model * wb[w.w_dtype]
    pred = (w.rank * w.d_model + w.d_ff * w.rank) * wb[w.p_dtype]
    return int(ffn + pred)
