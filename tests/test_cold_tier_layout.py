"""Host-side layout of the hybrid cold tier (no GPU): for dense and packed
records of every activation and weight dtype, row j >= hot of each matrix
read at cold + (j - hot) * stride (the addressing the kernels use) holds the
same bytes as row j of the original buffer, codes and Q4_0 scales alike."""
import ctypes

import numpy as np
import pytest
import torch

from activation_sparse_predictor_b200 import pi, synth
from helpers import small_workload


def _tensors(w):
    t = synth.layer_host(w, 0)
    out = {}
    for k in ("w_gate", "w_up", "w_down_t"):
        if k in t:
            v = t[k]
            if isinstance(v, tuple):
                out[k] = (torch.from_numpy(np.ascontiguousarray(v[0])),
                          torch.from_numpy(np.ascontiguousarray(v[1]).view(np.float16)))
            else:
                out[k] = torch.from_numpy(np.ascontiguousarray(v))
    for k in ("bias", "p1", "p2", "p_bias"):
        out[k] = torch.from_numpy(np.ascontiguousarray(t[k]))
    return out


def _strides(L):
    c = L.c
    up = c.w_up_row_stride or c.w_row_stride
    return {"w_gate": c.w_row_stride, "w_up": up if L.act == "reglu" else c.w_row_stride,
            "w_down_t": c.w_down_row_stride}


@pytest.mark.parametrize("act", ["relu", "reglu", "relu2"])
@pytest.mark.parametrize("wdt", ["f32", "f16", "q4_0"])
@pytest.mark.parametrize("packed", [False, True])
@pytest.mark.parametrize("hot", [0, 40, 100])
def test_cold_rows_sit_where_the_kernels_read_them(act, wdt, packed, hot):
    w = small_workload(act, wdt, "f32" if wdt == "f32" else "f16", d=64, F=100, r=16, hot=hot)
    t = _tensors(w)
    L = pi.Layer.packed(w, t) if packed else pi.Layer.from_workload(w, t)
    Lc = L.with_host_cold_tier(pin=False)
    d = w.d_model
    codes = {"f32": 4 * d, "f16": 2 * d, "q4_0": d // 2}[wdt]
    sc = d // 16 if wdt == "q4_0" else 0
    strides = _strides(L)
    names = ("w_gate", "w_up", "w_down_t") if act == "reglu" else ("w_up", "w_down_t")
    for name in names:
        st = strides[name] or codes
        sst = strides[name] or sc
        hot_p, cold_p = getattr(L.c, name), getattr(Lc.c, name + "_cold")
        if hot == w.d_ff:  # no cold rows: no cold tier (the descriptor's pointers stay null)
            assert not cold_p
            continue
        assert cold_p and cold_p % 16 == 0 and getattr(Lc.c, name) == hot_p
        for j in range(hot, w.d_ff):
            got = ctypes.string_at(cold_p + (j - hot) * st, codes)
            assert got == ctypes.string_at(hot_p + j * st, codes), (name, j)
        if wdt == "q4_0":
            hs = getattr(L.c, name + "_scales")
            cs = getattr(Lc.c, name + "_cold_scales")
            assert cs and cs % 2 == 0
            for j in range(hot, w.d_ff):
                got = ctypes.string_at(cs + (j - hot) * sst, sc)
                assert got == ctypes.string_at(hs + j * sst, sc), (name, "scales", j)
    if act != "reglu":
        assert not Lc.c.w_gate_cold
