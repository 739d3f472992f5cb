"""Thin ctypes binding of libpi.so (declared in include/pi.h).

Argument marshalling only: every step of the path runs in the library's
CUDA kernels.  Tensors are torch CUDA tensors (torch supplies device memory
and streams); functions carry the C names.  Importing this module without the
built library raises, so nothing can silently fall back to another path.
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpi.so")
PI_PREDICT_NOALLOC_MAX_FLOATS = 262144  # include/pi.h
HEADER = os.path.join(os.path.dirname(_HERE), "include", "pi.h")

PI_OK, PI_ERR_INVALID, PI_ERR_UNSUPPORTED, PI_ERR_CUDA, PI_ERR_TIMEOUT, PI_ERR_DEVICE_CHECK = range(6)
PI_F32, PI_F16, PI_Q4_0 = 0, 1, 2
PI_RELU, PI_REGLU, PI_RELU2 = 0, 1, 2
PI_MASK_PER_TOKEN, PI_MASK_UNION = 0, 1
DTYPES = {"f32": PI_F32, "f16": PI_F16, "q4_0": PI_Q4_0}
ACTS = {"relu": PI_RELU, "reglu": PI_REGLU, "relu2": PI_RELU2}
MODES = {"per_token": PI_MASK_PER_TOKEN, "union": PI_MASK_UNION}


class PiError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_status_name(status)}: {msg}")
        self.status = status


class pi_layer(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("rank", ctypes.c_int32),
        ("hot", ctypes.c_int32), ("act", ctypes.c_int32), ("w_dtype", ctypes.c_int32),
        ("p_dtype", ctypes.c_int32),
        ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down_t", ctypes.c_void_p),
        ("w_gate_scales", ctypes.c_void_p), ("w_up_scales", ctypes.c_void_p),
        ("w_down_t_scales", ctypes.c_void_p), ("bias", ctypes.c_void_p),
        ("p1", ctypes.c_void_p), ("p2", ctypes.c_void_p), ("p_bias", ctypes.c_void_p),
        ("w_row_stride", ctypes.c_int64), ("w_down_row_stride", ctypes.c_int64),
        ("w_up_row_stride", ctypes.c_int64),
        ("w_gate_cold", ctypes.c_void_p), ("w_up_cold", ctypes.c_void_p),
        ("w_down_t_cold", ctypes.c_void_p), ("w_gate_cold_scales", ctypes.c_void_p),
        ("w_up_cold_scales", ctypes.c_void_p), ("w_down_t_cold_scales", ctypes.c_void_p),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libpi.so is not built ({LIB_PATH}); run __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    L = ctypes.POINTER(pi_layer)
    sig = {
        "pi_workspace_bytes": (sz, [L, i32, i32]),
        "pi_workspace_init": (i32, [vp, sz, vp]),
        "pi_predict": (i32, [L, vp, i32, f32, vp, vp, sz, vp]),
        "pi_predict_noalloc": (i32, [L, vp, i32, f32, vp, vp]),
        "pi_compact": (i32, [vp, i32, i32, i32, i32, vp, vp, vp]),
        "pi_sparse_ffn": (i32, [L, vp, i32, vp, vp, vp, i32, vp, vp, sz, vp]),
        "pi_ffn_stack": (i32, [L, i32, vp, i32, f32, i32, vp, vp, sz, vp]),
        "pi_get_device_status": (i32, [vp, vp, i32, ctypes.POINTER(ctypes.c_uint32)]),
        "pi_ffn_stack_profile": (i32, [L, i32, vp, i32, f32, i32, vp, vp, sz, vp,
                                       ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)]),
        "pi_kind_name": (ctypes.c_char_p, [i32]),
        "pi_read_counters": (i32, [vp, vp, i32, ctypes.POINTER(ctypes.c_uint64)]),
        "pi_read_cold_counters": (i32, [vp, vp, i32, ctypes.POINTER(ctypes.c_uint64)]),
        "pi_read_list": (i32, [L, i32, i32, vp, sz, vp, ctypes.POINTER(ctypes.c_int32), i32,
                               ctypes.POINTER(ctypes.c_int32)]),
        "pi_ffn_stack_timeline": (i32, [L, i32, vp, f32, vp, sz, vp, vp, vp]),
        "pi_device_sms": (i32, []),
        "pi_kernel_launches": (ctypes.c_ulonglong, []),
        "pi_wait_selftest": (i32, [vp, sz, i32, ctypes.c_uint, vp]),
        "pi_status_string": (ctypes.c_char_p, [i32]),
        "pi_last_error": (ctypes.c_char_p, []),
        "pi_version": (i32, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


_lib = _load()


def declared_functions(header: str = HEADER) -> list[str]:
    """Names of the functions include/pi.h declares."""
    src = open(header).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pi_[a-z_]+)\s*\(", src)))


def _status_name(st: int) -> str:
    return _lib.pi_status_string(st).decode()


def _check(st: int) -> None:
    if st != PI_OK:
        raise PiError(st, _lib.pi_last_error().decode())


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream, device=None):
    import torch
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


# ------------------------------------------------------------------ layers

class Layer:
    """A pi_layer descriptor over torch device tensors (kept alive here).

    `tensors` keys: w_gate (ReGLU), w_up, w_down_t (tensors, or (codes,
    scales) pairs for q4_0), bias, p1, p2, p_bias."""

    def __init__(self, *, d_model, d_ff, rank, hot, act, w_dtype, p_dtype, tensors: dict,
                 w_row_stride: int = 0, w_down_row_stride: int = 0, w_up_row_stride: int = 0):
        self.tensors = tensors
        self.d_model, self.d_ff, self.rank, self.hot = d_model, d_ff, rank, hot
        self.act, self.w_dtype, self.p_dtype = act, w_dtype, p_dtype

        def w(name):
            v = tensors.get(name)
            if v is None:
                return None, None
            if isinstance(v, tuple):
                return _ptr(v[0]), _ptr(v[1])
            return _ptr(v), None

        g, gs = w("w_gate")
        u, us = w("w_up")
        dn, ds = w("w_down_t")
        self.c = pi_layer(d_model, d_ff, rank, hot, ACTS[act], DTYPES[w_dtype], DTYPES[p_dtype],
                          g, u, dn, gs, us, ds, _ptr(tensors.get("bias")), _ptr(tensors["p1"]),
                          _ptr(tensors["p2"]), _ptr(tensors.get("p_bias")), w_row_stride,
                          w_down_row_stride, w_up_row_stride)

    @classmethod
    def from_workload(cls, w, tensors: dict, **strides) -> "Layer":
        return cls(d_model=w.d_model, d_ff=w.d_ff, rank=w.rank, hot=w.hot, act=w.act,
                   w_dtype=w.w_dtype, p_dtype=w.p_dtype, tensors=tensors, **strides)

    @classmethod
    def packed(cls, w, tensors: dict) -> "Layer":
        """A layer whose neuron records are packed (see pack_records) the way
        the single-token kernel reads them.  Returns the Layer; the packed
        buffers live in it."""
        packed, strides = pack_records(w, tensors)
        return cls.from_workload(w, packed, **strides)

    @property
    def words(self) -> int:
        return (self.d_ff + 31) // 32

    def with_host_cold_tier(self, pin: bool = True) -> "Layer":
        """The same layer with rows [hot, d_ff) of w_gate / w_up / w_down_t
        (and their Q4_0 scales) read from page-locked host memory: each
        weight buffer's rows from `hot` on are copied to a pinned host
        buffer with the same row layout, and the descriptor's cold pointers
        point into it (see pi_layer).  The device tensors are shared with
        this layer; the returned layer never reads their rows >= hot.
        (pin=False leaves the copies in pageable memory, which the library
        rejects: for checking the layout without a GPU.)"""
        import torch
        if self.hot >= self.d_ff:
            return self  # no cold rows: nothing to move
        bufs, host = {}, {}

        def base_of(t):  # the row-major buffer a weight view lives in
            b = t
            while b._base is not None:
                b = b._base
            return b

        def cold_ptr(t):
            if t is None:
                return None
            b = base_of(t)
            rows = b.reshape(self.d_ff, -1)
            assert rows.shape[0] == self.d_ff and b.is_contiguous(), "one row per neuron"
            key = b.data_ptr()
            if key not in host:
                h = torch.empty((rows.shape[0] - self.hot, rows.shape[1]), dtype=rows.dtype,
                                pin_memory=pin)
                h.copy_(rows[self.hot:])
                host[key] = h
                bufs[key] = rows
            rs = bufs[key].stride(0) * bufs[key].element_size()
            off = t.data_ptr() - key  # offset inside the first row
            assert 0 <= off < rs and t.stride(0) * t.element_size() == rs, "rows must share the buffer's stride"
            return host[key].data_ptr() + off

        out = Layer.__new__(Layer)
        out.__dict__.update(self.__dict__)
        c = pi_layer()
        ctypes.pointer(c)[0] = self.c
        for name, fld, sfld in (("w_gate", "w_gate_cold", "w_gate_cold_scales"),
                                ("w_up", "w_up_cold", "w_up_cold_scales"),
                                ("w_down_t", "w_down_t_cold", "w_down_t_cold_scales")):
            v = self.tensors.get(name)
            if v is None:
                continue
            codes, scales = v if isinstance(v, tuple) else (v, None)
            setattr(c, fld, cold_ptr(codes))
            if scales is not None:
                setattr(c, sfld, cold_ptr(scales))
        out.c = c
        out.cold_host = host  # keeps the pinned buffers alive
        return out


def pack_records(w, tensors: dict):
    """Rearranges a layer's FFN weights (dense matrices as produced by the
    input generator) into per-neuron records on the same device, each row as
    [codes | scales] for Q4_0, padded to 16 bytes:
      ReGLU : gate records one after another (a neuron's activity is decided
              by its gate row alone), and per neuron [up row | down row] (read
              together, only for neurons whose gate fires);
      ReLU, squared ReLU: up records, and down records, one after another.
    Returns (tensor dict with views into the packed buffers, strides)."""
    import torch
    def q4rows(pair):
        codes, scales = pair
        F = codes.shape[0]
        return torch.cat([codes.reshape(F, -1), scales.contiguous().view(torch.uint8).reshape(F, -1)], 1)
    def pad16(b):  # each record a multiple of 16 bytes (16-byte aligned rows)
        extra = (-b.shape[1]) % 16
        return b if extra == 0 else torch.cat([b, b.new_zeros((b.shape[0], extra))], 1)
    def asbytes(t):
        b = q4rows(t) if isinstance(t, tuple) else t.contiguous().view(torch.uint8).reshape(t.shape[0], -1)
        return pad16(b)
    out = {k: v for k, v in tensors.items() if k not in ("w_gate", "w_up", "w_down_t")}
    rb = {"f32": 4 * w.d_model, "f16": 2 * w.d_model, "q4_0": w.d_model // 2}[w.w_dtype]
    sc = w.d_model // 16 if w.w_dtype == "q4_0" else 0
    rec = rb + sc + (-(rb + sc)) % 16
    def rows(buf, off):
        if w.w_dtype == "q4_0":
            return (buf[:, off:off + rb], buf[:, off + rb:off + rb + sc])
        return buf[:, off:off + rb]
    if w.act == "reglu":
        first = asbytes(tensors["w_gate"]).contiguous()
        second = torch.cat([asbytes(tensors["w_up"]), asbytes(tensors["w_down_t"])], 1).contiguous()
        out["w_gate"], out["w_up"], out["w_down_t"] = rows(first, 0), rows(second, 0), rows(second, rec)
        strides = {"w_row_stride": rec, "w_up_row_stride": 2 * rec, "w_down_row_stride": 2 * rec}
    else:
        first = asbytes(tensors["w_up"]).contiguous()
        second = asbytes(tensors["w_down_t"]).contiguous()
        out["w_up"], out["w_down_t"] = rows(first, 0), rows(second, 0)
        strides = {"w_row_stride": rec, "w_down_row_stride": rec}
    out["_packed_first"], out["_packed_second"] = first, second
    return out, strides


def _layer_array(layers):
    arr = (pi_layer * len(layers))()
    for i, L in enumerate(layers):
        arr[i] = L.c
    return arr


# -------------------------------------------------------------- entry points

def pi_workspace_bytes(layers, batch: int) -> int:
    layers = layers if isinstance(layers, (list, tuple)) else [layers]
    n = _lib.pi_workspace_bytes(_layer_array(layers), len(layers), batch)
    if n == 0:
        raise PiError(PI_ERR_INVALID, "invalid layers or batch for workspace sizing")
    return int(n)


def pi_workspace_init(ws, stream=None) -> None:
    _check(_lib.pi_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))


def workspace(layers, batch: int, device="cuda", stream=None):
    """Allocate (with torch) and initialise a workspace for these layers."""
    import torch
    n = pi_workspace_bytes(layers, batch)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    pi_workspace_init(ws, stream)
    return ws


def pi_predict(layer: Layer, xh, tau: float, mask=None, ws=None, stream=None):
    """Predicted masks [batch][words] (uint32 as int32 tensor) of FFN inputs xh."""
    import torch
    batch = xh.shape[0]
    if mask is None:
        mask = torch.empty((batch, layer.words), dtype=torch.int32, device=xh.device)
    if ws is None:
        ws = workspace([layer], batch, xh.device, stream)
    _check(_lib.pi_predict(ctypes.byref(layer.c), _ptr(xh), batch, tau, _ptr(mask), _ptr(ws),
                           ws.numel(), _stream(stream)))
    return mask


def pi_predict_noalloc(layer: Layer, xh, tau: float, mask, stream=None):
    """The predictor without a workspace: u lives in the library's static
    per-device buffer (batch * rank <= PI_PREDICT_NOALLOC_MAX_FLOATS), so the
    call allocates nothing; `mask` [batch][words] int32 is the caller's.
    Always the CUDA-core predictor kernels (see include/pi.h).  Calls whose
    GPU work overlaps on one device race on that buffer."""
    import torch
    batch = xh.shape[0]
    if (tuple(mask.shape) != (batch, layer.words) or mask.dtype != torch.int32
            or not mask.is_contiguous() or mask.device != xh.device):
        raise ValueError(f"mask must be a contiguous int32 tensor of shape {(batch, layer.words)} "
                         f"on {xh.device}")
    if xh.dtype != torch.float32 or not xh.is_contiguous() or xh.dim() != 2 \
            or xh.shape[1] != layer.d_model:
        raise ValueError(f"xh must be a contiguous float32 tensor [batch][{layer.d_model}]")
    _check(_lib.pi_predict_noalloc(ctypes.byref(layer.c), _ptr(xh), batch, tau,
                                   _ptr(mask), _stream(stream)))
    return mask


def pi_compact(mask, d_ff: int, begin: int, mode: int, idx=None, count=None, stream=None):
    """(idx, count) device tensors of the ascending active lists."""
    import torch
    batch = mask.shape[0]
    lists = 1 if mode == PI_MASK_UNION else batch
    if idx is None:
        idx = torch.empty((lists, d_ff), dtype=torch.int32, device=mask.device)
    if count is None:
        count = torch.empty(lists, dtype=torch.int32, device=mask.device)
    _check(_lib.pi_compact(_ptr(mask), batch, d_ff, begin, mode, _ptr(idx), _ptr(count),
                           _stream(stream)))
    return idx, count


def pi_sparse_ffn(layer: Layer, xh, mask, idx, count, mode: int, y=None, ws=None, stream=None):
    """y [batch][d] of the FFN over [0, hot) U idx[:count]."""
    import torch
    batch = xh.shape[0]
    if y is None:
        y = torch.empty((batch, layer.d_model), dtype=torch.float32, device=xh.device)
    if ws is None:
        ws = workspace([layer], batch, xh.device, stream)
    _check(_lib.pi_sparse_ffn(ctypes.byref(layer.c), _ptr(xh), batch, _ptr(mask), _ptr(idx),
                              _ptr(count), mode, _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))
    return y


def pi_ffn_stack(layers, x, tau: float, mode: int, mask_trace=None, ws=None, stream=None,
                 _arr=None):
    """Runs the stack on x [batch][d] in place; returns x."""
    batch = x.shape[0]
    if ws is None:
        ws = workspace(layers, batch, x.device, stream)
    arr = _arr if _arr is not None else _layer_array(layers)
    _check(_lib.pi_ffn_stack(arr, len(layers), _ptr(x), batch, tau, mode, _ptr(mask_trace),
                             _ptr(ws), ws.numel(), _stream(stream)))
    return x


PI_KINDS = 8


def pi_ffn_stack_profile(layers, x, tau: float, mode: int, mask_trace=None, ws=None,
                         stream=None, _arr=None):
    """pi_ffn_stack with CUDA events around every launch: returns
    {kind name: (total ms, launches)}; synchronises the stream."""
    batch = x.shape[0]
    if ws is None:
        ws = workspace(layers, batch, x.device, stream)
    arr = _arr if _arr is not None else _layer_array(layers)
    ms = (ctypes.c_float * PI_KINDS)()
    n = (ctypes.c_int * PI_KINDS)()
    _check(_lib.pi_ffn_stack_profile(arr, len(layers), _ptr(x), batch, tau, mode,
                                     _ptr(mask_trace), _ptr(ws), ws.numel(), _stream(stream),
                                     ms, n))
    return {_lib.pi_kind_name(k).decode(): (float(ms[k]), int(n[k])) for k in range(PI_KINDS)}


def pi_read_cold_counters(ws, clear: bool = False, stream=None):
    """(first-matrix rows, w_down_t rows, ReGLU w_up rows) read from a host-memory cold tier."""
    out = (ctypes.c_uint64 * 3)()
    _check(_lib.pi_read_cold_counters(_ptr(ws), _stream(stream), int(clear), out))
    return int(out[0]), int(out[1]), int(out[2])


def pi_read_counters(ws, clear: bool = False, stream=None):
    """(first-matrix rows read, w_down_t rows read, ReGLU w_up rows read);
    synchronises the stream (include/pi.h)."""
    out = (ctypes.c_uint64 * 3)()
    _check(_lib.pi_read_counters(_ptr(ws), _stream(stream), int(clear), out))
    return int(out[0]), int(out[1]), int(out[2])


def pi_read_list(layers, batch: int, ws, stream=None, _arr=None):
    """The ascending cold list (numpy int32) of the last layer of the last
    stack call on `ws` (include/pi.h); synchronises the stream."""
    import numpy as np
    layers = layers if isinstance(layers, (list, tuple)) else [layers]
    arr = _arr if _arr is not None else _layer_array(layers)
    cap = max(L.d_ff for L in layers)
    out = (ctypes.c_int32 * cap)()
    n = ctypes.c_int32(0)
    _check(_lib.pi_read_list(arr, len(layers), batch, _ptr(ws), ws.numel(), _stream(stream),
                             out, cap, ctypes.byref(n)))
    return np.frombuffer(out, dtype=np.int32, count=int(n.value)).copy()


def pi_ffn_stack_timeline(layers, x, tau: float, ws=None, stream=None, _arr=None):
    """Runs the stack (batch 1, persistent kernel) and returns (timeline
    [n_layers][SMs][16], unit timeline [n_layers][512][4]) as device int64
    tensors (see include/pi.h)."""
    import torch
    if ws is None:
        ws = workspace(layers, 1, x.device, stream)
    arr = _arr if _arr is not None else _layer_array(layers)
    tl = torch.zeros((len(layers), pi_device_sms(), 16), dtype=torch.int64, device=x.device)
    ut = torch.zeros((len(layers), 512, 4), dtype=torch.int64, device=x.device)
    _check(_lib.pi_ffn_stack_timeline(arr, len(layers), _ptr(x), tau, _ptr(ws), ws.numel(),
                                      _stream(stream), _ptr(tl), _ptr(ut)))
    return tl, ut


def pi_device_sms() -> int:
    return int(_lib.pi_device_sms())


def pi_kernel_launches() -> int:
    """Kernels launched by the library in this process so far (include/pi.h)."""
    return int(_lib.pi_kernel_launches())


def pi_kind_name(kind: int) -> str:
    return _lib.pi_kind_name(kind).decode()


def pi_get_device_status(ws, clear: bool = False, stream=None):
    """(status, raw word); synchronises the stream."""
    word = ctypes.c_uint32(0)
    st = _lib.pi_get_device_status(_ptr(ws), _stream(stream), int(clear), ctypes.byref(word))
    return st, int(word.value)


def pi_wait_selftest(ws, kind: int, timeout_us: int, stream=None) -> None:
    """Runs the fused kernel's bounded wait on a wait nothing completes (kind
    0: mbarrier, 1: grid barrier) for timeout_us; the timeout shows in
    pi_get_device_status."""
    _check(_lib.pi_wait_selftest(_ptr(ws), ws.numel(), kind, timeout_us, _stream(stream)))


def pi_status_string(st: int) -> str:
    return _status_name(st)


def pi_last_error() -> str:
    return _lib.pi_last_error().decode()


def pi_version() -> int:
    return int(_lib.pi_version())


def layer_array(layers):
    """A reusable C array of descriptors for pi_ffn_stack(..., _arr=...)."""
    return _layer_array(layers)


def library_path() -> str:
    return LIB_PATH
