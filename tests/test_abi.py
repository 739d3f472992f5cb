"""The C-ABI library loads and exports every function include/pi.h declares;
host-side argument validation rejects bad calls before enqueuing anything.
CPU only: no call here reaches a kernel launch."""
import ctypes
import subprocess

import pytest

from activation_sparse_predictor_b200 import build


@pytest.fixture(scope="module")
def pi():
    build.build_libpi()
    from activation_sparse_predictor_b200 import pi as m
    return m


def test_header_declares_the_boundary(pi):
    names = pi.declared_functions()
    for required in ("pi_predict", "pi_compact", "pi_sparse_ffn", "pi_ffn_stack",
                     "pi_workspace_bytes", "pi_get_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol(pi):
    lib = ctypes.CDLL(pi.LIB_PATH)
    out = subprocess.run(["nm", "-D", "--defined-only", pi.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in pi.declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_library_is_sm100a_only(pi):
    out = subprocess.run(["cuobjdump", "--list-elf", pi.LIB_PATH], capture_output=True,
                         text=True).stdout
    archs = {tok for tok in out.split() if "sm_" in tok}
    assert archs and all("sm_100a" in a for a in archs), archs


def test_status_strings_and_version(pi):
    assert pi.pi_version() == 3
    assert pi.pi_status_string(pi.PI_OK) == "PI_OK"
    assert pi.pi_status_string(pi.PI_ERR_TIMEOUT) == "PI_ERR_TIMEOUT"
    assert pi.pi_status_string(99) == "PI_ERR_UNKNOWN"


def test_kernel_launch_counter_without_gpu(pi):
    a = pi.pi_kernel_launches()
    b = pi.pi_kernel_launches()
    assert isinstance(a, int) and 0 <= a <= b


FAKE = 1 << 20  # an aligned, never-dereferenced address


def _layer(pi, **over):
    base = dict(d_model=64, d_ff=256, rank=16, hot=32, act=pi.PI_RELU, w_dtype=pi.PI_F16,
                p_dtype=pi.PI_F16)
    kw = dict(base)
    kw.update({k: v for k, v in over.items() if k in base})
    c = pi.pi_layer(kw["d_model"], kw["d_ff"], kw["rank"], kw["hot"], kw["act"], kw["w_dtype"],
                    kw["p_dtype"], FAKE if kw["act"] == pi.PI_REGLU else None, FAKE, FAKE,
                    FAKE if kw["w_dtype"] == pi.PI_Q4_0 else None,
                    FAKE if kw["w_dtype"] == pi.PI_Q4_0 else None,
                    FAKE if kw["w_dtype"] == pi.PI_Q4_0 else None, FAKE, FAKE, FAKE, FAKE)
    for k, v in over.items():
        if k not in base:
            setattr(c, k, v)
    return c


@pytest.mark.parametrize("over,expect", [
    (dict(d_model=0), "PI_ERR_INVALID"),
    (dict(d_model=20000), "PI_ERR_INVALID"),
    (dict(d_ff=0), "PI_ERR_INVALID"),
    (dict(hot=300), "PI_ERR_INVALID"),
    (dict(hot=-1), "PI_ERR_INVALID"),
    (dict(rank=12), "PI_ERR_INVALID"),          # f16 predictor needs rank % 8
    (dict(d_model=60), "PI_ERR_INVALID"),       # not a multiple of 8
    (dict(w_dtype=2, d_model=48), "PI_ERR_INVALID"),  # Q4_0 needs d % 32
    (dict(act=7), "PI_ERR_INVALID"),
    (dict(w_dtype=9), "PI_ERR_INVALID"),
    (dict(p_dtype=2), "PI_ERR_UNSUPPORTED"),
    (dict(w_up=None), "PI_ERR_INVALID"),
    (dict(w_up=FAKE + 4), "PI_ERR_INVALID"),    # misaligned weight
    (dict(act=1, w_gate=None), "PI_ERR_INVALID"),
    (dict(w_dtype=2, d_model=64, w_up_scales=None), "PI_ERR_INVALID"),
    (dict(w_up_row_stride=256), "PI_ERR_INVALID"),        # a ReGLU-only field on ReLU
    (dict(act=1, w_up_row_stride=100), "PI_ERR_INVALID"),  # not a multiple of 16
    (dict(act=1, w_up_row_stride=64), "PI_ERR_INVALID"),   # shorter than one row (128 B)
])
def test_layer_validation(pi, over, expect):
    L = _layer(pi, **over)
    st = pi._lib.pi_predict(ctypes.byref(L), FAKE, 1, 0.5, FAKE, FAKE, 1 << 30, None)
    assert pi.pi_status_string(st) == expect, pi.pi_last_error()
    assert pi.pi_last_error()


def test_call_validation(pi):
    L = _layer(pi)
    lib = pi._lib
    # batch out of range, tau out of range, misaligned input, small workspace
    assert lib.pi_predict(ctypes.byref(L), FAKE, 0, 0.5, FAKE, FAKE, 1 << 30, None) == pi.PI_ERR_INVALID
    assert lib.pi_predict(ctypes.byref(L), FAKE, 65, 0.5, FAKE, FAKE, 1 << 30, None) == pi.PI_ERR_INVALID
    assert lib.pi_predict(ctypes.byref(L), FAKE, 1, 1.0, FAKE, FAKE, 1 << 30, None) == pi.PI_ERR_INVALID
    assert lib.pi_predict(ctypes.byref(L), FAKE + 8, 1, 0.5, FAKE, FAKE, 1 << 30, None) == pi.PI_ERR_INVALID
    assert lib.pi_predict(ctypes.byref(L), FAKE, 1, 0.5, FAKE, FAKE, 64, None) == pi.PI_ERR_INVALID
    assert "workspace too small" in pi.pi_last_error()
    assert lib.pi_predict(ctypes.byref(L), FAKE, 1, 0.5, FAKE, FAKE + 16, 1 << 30, None) == pi.PI_ERR_INVALID
    # compaction arguments
    assert lib.pi_compact(FAKE, 1, 0, 0, 1, FAKE, FAKE, None) == pi.PI_ERR_INVALID
    assert lib.pi_compact(FAKE, 1, 100, 101, 1, FAKE, FAKE, None) == pi.PI_ERR_INVALID
    assert lib.pi_compact(FAKE, 1, 100, 0, 5, FAKE, FAKE, None) == pi.PI_ERR_INVALID
    assert lib.pi_compact(None, 1, 100, 0, 1, FAKE, FAKE, None) == pi.PI_ERR_INVALID
    # sparse FFN: per-token mode with batch > 1 needs the mask
    assert lib.pi_sparse_ffn(ctypes.byref(L), FAKE, 2, None, FAKE, FAKE, 0, FAKE, FAKE, 1 << 30,
                             None) == pi.PI_ERR_INVALID
    # stack: layers must share d_model / d_ff
    arr = (pi.pi_layer * 2)(_layer(pi), _layer(pi, d_ff=512))
    assert lib.pi_ffn_stack(arr, 2, FAKE, 1, 0.5, 1, None, FAKE, 1 << 30, None) == pi.PI_ERR_INVALID
    assert "share" in pi.pi_last_error()
    assert lib.pi_ffn_stack(arr, 0, FAKE, 1, 0.5, 1, None, FAKE, 1 << 30, None) == pi.PI_ERR_INVALID
    assert lib.pi_workspace_bytes(arr, 2, 0) == 0
    assert lib.pi_workspace_init(FAKE + 8, 1024, None) == pi.PI_ERR_INVALID


def test_newer_entry_points_validate_before_enqueuing(pi):
    lib = pi._lib
    L = _layer(pi)
    # pi_predict_noalloc: its static scratch holds batch x rank <= 262144 floats
    big = _layer(pi, rank=8192)
    assert lib.pi_predict_noalloc(ctypes.byref(big), FAKE, 64, 0.5, FAKE, None) == pi.PI_ERR_INVALID
    assert "static scratch" in pi.pi_last_error()
    assert lib.pi_predict_noalloc(ctypes.byref(L), FAKE, 0, 0.5, FAKE, None) == pi.PI_ERR_INVALID
    assert lib.pi_predict_noalloc(ctypes.byref(L), FAKE, 1, 0.0, FAKE, None) == pi.PI_ERR_INVALID
    assert lib.pi_predict_noalloc(ctypes.byref(L), FAKE + 4, 1, 0.5, FAKE, None) == pi.PI_ERR_INVALID
    assert lib.pi_predict_noalloc(ctypes.byref(L), FAKE, 1, 0.5, None, None) == pi.PI_ERR_INVALID
    # pi_wait_selftest: workspace, wait kind and time limit
    assert lib.pi_wait_selftest(None, 4096, 0, 2000, None) == pi.PI_ERR_INVALID
    assert lib.pi_wait_selftest(FAKE + 8, 4096, 0, 2000, None) == pi.PI_ERR_INVALID
    assert lib.pi_wait_selftest(FAKE, 16, 0, 2000, None) == pi.PI_ERR_INVALID
    assert lib.pi_wait_selftest(FAKE, 4096, 2, 2000, None) == pi.PI_ERR_INVALID
    assert lib.pi_wait_selftest(FAKE, 4096, 1, 0, None) == pi.PI_ERR_INVALID
    assert lib.pi_wait_selftest(FAKE, 4096, 1, 20000000, None) == pi.PI_ERR_INVALID
    # counters and the timeline need their buffers
    out = (ctypes.c_uint64 * 2)()
    assert lib.pi_read_counters(None, None, 0, out) == pi.PI_ERR_INVALID
    assert lib.pi_read_counters(FAKE, None, 0, None) == pi.PI_ERR_INVALID
    arr = (pi.pi_layer * 1)(L)
    assert lib.pi_ffn_stack_timeline(arr, 1, FAKE, 0.5, FAKE, 1 << 30, None, None,
                                     None) == pi.PI_ERR_INVALID
    assert lib.pi_ffn_stack_timeline(arr, 0, FAKE, 0.5, FAKE, 1 << 30, None, FAKE,
                                     None) == pi.PI_ERR_INVALID
    # pi_read_list: layers, batch, outputs and the workspace size
    n = ctypes.c_int32(0)
    idx = (ctypes.c_int32 * 8)()
    assert lib.pi_read_list(arr, 0, 1, FAKE, 1 << 30, None, idx, 8, ctypes.byref(n)) == pi.PI_ERR_INVALID
    assert lib.pi_read_list(arr, 1, 65, FAKE, 1 << 30, None, idx, 8, ctypes.byref(n)) == pi.PI_ERR_INVALID
    assert lib.pi_read_list(arr, 1, 1, FAKE, 1 << 30, None, idx, 8, None) == pi.PI_ERR_INVALID
    assert lib.pi_read_list(arr, 1, 1, FAKE, 1 << 30, None, None, 8, ctypes.byref(n)) == pi.PI_ERR_INVALID
    assert lib.pi_read_list(arr, 1, 1, FAKE, 1 << 30, None, idx, -1, ctypes.byref(n)) == pi.PI_ERR_INVALID
    assert lib.pi_read_list(arr, 1, 1, FAKE, 64, None, idx, 8, ctypes.byref(n)) == pi.PI_ERR_INVALID
    assert "too small" in pi.pi_last_error()
    assert lib.pi_read_list(arr, 1, 1, FAKE + 8, 1 << 30, None, idx, 8, ctypes.byref(n)) == pi.PI_ERR_INVALID


def test_workspace_grows_with_batch(pi):
    L = _layer(pi)
    arr = (pi.pi_layer * 1)(L)
    a = pi._lib.pi_workspace_bytes(arr, 1, 1)
    b = pi._lib.pi_workspace_bytes(arr, 1, 16)
    assert 0 < a < b
    assert a % 256 == 0


def test_layer_struct_matches_the_header(pi, tmp_path):
    """ctypes' pi_layer has the C struct's size and field offsets (the
    cold-tier pointers at the end included)."""
    import os
    fields = [f for f, _ in pi.pi_layer._fields_]
    src = tmp_path / "layout.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"pi.h\"\nint main(void) {\n"
                   "  printf(\"%zu\\n\", sizeof(pi_layer));\n" +
                   "".join(f"  printf(\"%zu\\n\", offsetof(pi_layer, {f}));\n" for f in fields) +
                   "  return 0;\n}\n")
    exe = tmp_path / "layout"
    inc = os.path.join(os.path.dirname(pi.HEADER))
    subprocess.run(["gcc", "-std=c11", "-I", inc, str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    assert got[0] == ctypes.sizeof(pi.pi_layer)
    for f, off in zip(fields, got[1:]):
        assert getattr(pi.pi_layer, f).offset == off, f


def test_cold_tier_validation(pi):
    """A cold tier must be complete (w_gate_cold for ReGLU, scales for Q4_0)
    and aligned; checked before any device call."""
    for over in (dict(w_up_cold=FAKE),                                   # no w_down_t_cold
                 dict(act=1, w_up_cold=FAKE, w_down_t_cold=FAKE),        # ReGLU without gate
                 dict(w_dtype=2, d_model=64, w_up_cold=FAKE, w_down_t_cold=FAKE),  # no scales
                 dict(w_up_cold=FAKE + 4, w_down_t_cold=FAKE),           # misaligned
                 dict(w_up_cold_scales=FAKE)):                           # scales alone
        L = _layer(pi, **over)
        st = pi._lib.pi_predict(ctypes.byref(L), FAKE, 1, 0.5, FAKE, FAKE, 1 << 30, None)
        assert pi.pi_status_string(st) == "PI_ERR_INVALID", (over, pi.pi_last_error())
        assert "cold" in pi.pi_last_error()
