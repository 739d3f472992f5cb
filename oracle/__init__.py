"""CPU oracle of the predictor-gated sparse FFN (TEST INFRASTRUCTURE ONLY).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
binding) never does, and the two share no code: the only module both sides
use is the seeded input generator ``activation_sparse_predictor_b200.synth``.

The arithmetic lives in ``pi_oracle.c`` (plain C, double accumulation); this
module marshals numpy arrays.  Every function is pinned by tests that do not
reuse it (see ``tests/test_oracle_pins.py``).
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from .build import LIB_PATH, build as _build

OR_F32, OR_F16, OR_Q4_0 = 0, 1, 2
OR_RELU, OR_REGLU, OR_RELU2 = 0, 1, 2
_DT = {"f32": OR_F32, "f16": OR_F16, "q4_0": OR_Q4_0}
_ACT = {"relu": OR_RELU, "reglu": OR_REGLU, "relu2": OR_RELU2}


class _Layer(ctypes.Structure):
    _fields_ = [
        ("d", ctypes.c_int32), ("F", ctypes.c_int32), ("r", ctypes.c_int32),
        ("H", ctypes.c_int32), ("act", ctypes.c_int32), ("wdt", ctypes.c_int32),
        ("pdt", ctypes.c_int32),
        ("wg", ctypes.c_void_p), ("wu", ctypes.c_void_p), ("wd", ctypes.c_void_p),
        ("sg", ctypes.c_void_p), ("su", ctypes.c_void_p), ("sd", ctypes.c_void_p),
        ("bias", ctypes.c_void_p), ("p1", ctypes.c_void_p), ("p2", ctypes.c_void_p),
        ("pbias", ctypes.c_void_p),
    ]


_lib = None
_lib_path = None


def load(path: str | None = None):
    """Load (building if needed) the oracle library; `path` loads another build
    of the same source (used by the planted-mistake tests)."""
    global _lib, _lib_path
    if path is None:
        if _lib is not None and _lib_path == LIB_PATH:
            return _lib
        _build()
        path = LIB_PATH
    lib = ctypes.CDLL(path)
    vp, i32, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
    lib.or_num_threads.restype = i32
    lib.or_set_num_threads.argtypes = [i32]
    lib.or_half_to_double.restype = dbl
    lib.or_half_to_double.argtypes = [ctypes.c_uint16]
    lib.or_q4_0_weight.restype = dbl
    lib.or_q4_0_weight.argtypes = [vp, vp, i32, ctypes.c_long, i32]
    lib.or_decode_row.argtypes = [i32, vp, vp, i32, ctypes.c_long, vp]
    lib.or_rmsnorm.argtypes = [vp, i32, vp]
    lib.or_predict.argtypes = [vp, vp, vp, vp]
    lib.or_mask.argtypes = [vp, i32, i32, dbl, vp]
    lib.or_compact.restype = i32
    lib.or_compact.argtypes = [vp, i32, i32, i32, vp]
    lib.or_ffn.argtypes = [vp, vp, vp, vp, vp]
    lib.or_rowset.argtypes = [i32, i32, vp, i32, vp]
    lib.or_layer_forward.argtypes = [vp, vp, dbl, vp, vp, vp]
    if path == LIB_PATH:
        _lib, _lib_path = lib, path
    return lib


def _p(a):
    return None if a is None else a.ctypes.data


class Oracle:
    """Numpy-facing wrapper over one build of the oracle library."""

    def __init__(self, path: str | None = None):
        self.lib = load(path)

    def num_threads(self) -> int:
        return int(self.lib.or_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.or_set_num_threads(int(n))

    # ----------------------------------------------------------- layer struct
    def _layer(self, L: dict):
        """Build the C struct for a layer dict (see synth.layer_host)."""
        w = L["workload"] if "workload" in L else None
        meta = L.get("meta") or {}
        d = meta.get("d_model", w.d_model if w else None)
        F = meta.get("d_ff", w.d_ff if w else None)
        r = meta.get("rank", w.rank if w else None)
        H = meta.get("hot", w.hot if w else 0)
        act = meta.get("act", w.act if w else "relu")
        wdt = meta.get("w_dtype", w.w_dtype if w else "f32")
        pdt = meta.get("p_dtype", w.p_dtype if w else "f32")
        keep = []

        def mat(a):
            if a is None:
                return None, None
            if isinstance(a, tuple):
                qs = np.ascontiguousarray(a[0], dtype=np.uint8)
                sc = np.ascontiguousarray(a[1]).view(np.uint16)
                keep.extend([qs, sc])
                return qs.ctypes.data, sc.ctypes.data
            a = np.ascontiguousarray(a)
            if a.dtype == np.float16:
                a = a.view(np.uint16)
            keep.append(a)
            return a.ctypes.data, None

        wg, sg = mat(L.get("w_gate"))
        wu, su = mat(L["w_up"])
        wd, sd = mat(L["w_down_t"])
        p1, _ = mat(L["p1"])
        p2, _ = mat(L["p2"])
        bias = L.get("bias")
        pbias = L.get("p_bias")
        if bias is not None:
            bias = np.ascontiguousarray(bias, dtype=np.float32)
            keep.append(bias)
        if pbias is not None:
            pbias = np.ascontiguousarray(pbias, dtype=np.float32)
            keep.append(pbias)
        s = _Layer(d, F, r, H, _ACT[act], _DT[wdt], _DT[pdt], wg, wu, wd, sg, su, sd,
                   _p(bias), p1, p2, _p(pbias))
        return s, keep

    # ------------------------------------------------------------ primitives
    def half_to_double(self, bits: int) -> float:
        return float(self.lib.or_half_to_double(bits))

    def decode_matrix(self, a, dtype: str, cols: int) -> np.ndarray:
        """Whole matrix decoded to float64 (rows x cols)."""
        if isinstance(a, tuple):
            qs = np.ascontiguousarray(a[0], dtype=np.uint8)
            sc = np.ascontiguousarray(a[1]).view(np.uint16)
            rows, w, s = qs.shape[0], qs, sc
        else:
            w = np.ascontiguousarray(a)
            if w.dtype == np.float16:
                w = w.view(np.uint16)
            rows, s = w.shape[0], None
        out = np.empty((rows, cols), np.float64)
        for i in range(rows):
            self.lib.or_decode_row(_DT[dtype], w.ctypes.data, _p(s), cols, i,
                                   out[i].ctypes.data)
        return out

    def rmsnorm(self, x: np.ndarray) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty(x.shape[-1], np.float64)
        self.lib.or_rmsnorm(x.ctypes.data, x.shape[-1], out.ctypes.data)
        return out

    def predict(self, L: dict, xh: np.ndarray):
        """(u, z) for one token's FFN input xh (float64)."""
        s, keep = self._layer(L)
        xh = np.ascontiguousarray(xh, dtype=np.float64)
        u = np.empty(s.r, np.float64)
        z = np.empty(s.F, np.float64)
        self.lib.or_predict(ctypes.byref(s), xh.ctypes.data, u.ctypes.data, z.ctypes.data)
        return u, z

    def mask(self, z: np.ndarray, F: int, H: int, theta: float) -> np.ndarray:
        z = np.ascontiguousarray(z, dtype=np.float64)
        m = np.empty((F + 31) // 32, np.uint32)
        self.lib.or_mask(z.ctypes.data, F, H, theta, m.ctypes.data)
        return m

    def compact(self, masks: np.ndarray, F: int, begin: int) -> np.ndarray:
        """Ascending active list over the OR of masks [nmask][words]."""
        masks = np.ascontiguousarray(np.atleast_2d(masks), dtype=np.uint32)
        idx = np.empty(max(F, 1), np.int32)
        n = self.lib.or_compact(masks.ctypes.data, masks.shape[0], F, begin, idx.ctypes.data)
        return idx[:n].copy()

    def ffn(self, L: dict, xh: np.ndarray, rowset: np.ndarray):
        """(h, y) of the FFN restricted to rowset (bool/uint8 [F])."""
        s, keep = self._layer(L)
        xh = np.ascontiguousarray(xh, dtype=np.float64)
        rs = np.ascontiguousarray(rowset, dtype=np.uint8)
        h = np.empty(s.F, np.float64)
        y = np.empty(s.d, np.float64)
        self.lib.or_ffn(ctypes.byref(s), xh.ctypes.data, rs.ctypes.data, h.ctypes.data,
                        y.ctypes.data)
        return h, y

    def rowset(self, F: int, H: int, idx: np.ndarray) -> np.ndarray:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        rs = np.empty(F, np.uint8)
        self.lib.or_rowset(F, H, idx.ctypes.data, len(idx), rs.ctypes.data)
        return rs

    # ------------------------------------------------------------- composites
    def dense_ffn(self, L: dict, xh: np.ndarray) -> np.ndarray:
        F = self._layer(L)[0].F
        return self.ffn(L, xh, np.ones(F, np.uint8))[1]

    def sparse_ffn(self, L: dict, xh: np.ndarray, idx: np.ndarray, hot: int | None = None):
        """y of the FFN over S = [0, hot) U idx."""
        s, _ = self._layer(L)
        H = s.H if hot is None else hot
        return self.ffn(L, xh, self.rowset(s.F, H, idx))[1]

    def layer_forward(self, L: dict, x: np.ndarray, tau: float):
        """One stack layer for one token: (x_out float64, mask, z)."""
        s, keep = self._layer(L)
        x = np.ascontiguousarray(x, dtype=np.float32)
        xo = np.empty(s.d, np.float64)
        m = np.empty((s.F + 31) // 32, np.uint32)
        z = np.empty(s.F, np.float64)
        theta = float(np.float32(math.log(tau / (1.0 - tau))))
        self.lib.or_layer_forward(ctypes.byref(s), x.ctypes.data, theta, xo.ctypes.data,
                                  m.ctypes.data, z.ctypes.data)
        return xo, m, z


def rel_l2(a, ref) -> float:
    """||a - ref|| / ||ref||; 0 if both are zero, inf if only ref is zero."""
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    nr = float(np.linalg.norm(ref))
    nd = float(np.linalg.norm(a - ref))
    if nr == 0.0:
        return 0.0 if nd == 0.0 else math.inf
    return nd / nr
