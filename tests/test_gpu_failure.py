"""Failure detection without a GPU fault: the fused kernel's bounded waits,
run on a wait nothing completes (an mbarrier phase with no arrival, a grid
barrier target no CTA reaches), end by their limit, report PI_ERR_TIMEOUT
through the workspace status word, and leave the context and the workspace
usable.  Argument checks of the self-test run on CPU."""
import ctypes
import time

import numpy as np
import pytest

from activation_sparse_predictor_b200 import synth

FAKE = 1 << 20


def _pi():
    from activation_sparse_predictor_b200 import build
    build.build_libpi()
    from activation_sparse_predictor_b200 import pi
    return pi


def test_wait_selftest_argument_checks():
    pi = _pi()
    lib = pi._lib
    assert lib.pi_wait_selftest(None, 1 << 20, 0, 100, None) == pi.PI_ERR_INVALID
    assert lib.pi_wait_selftest(FAKE + 8, 1 << 20, 0, 100, None) == pi.PI_ERR_INVALID
    assert lib.pi_wait_selftest(FAKE, 64, 0, 100, None) == pi.PI_ERR_INVALID
    assert lib.pi_wait_selftest(FAKE, 1 << 20, 2, 100, None) == pi.PI_ERR_INVALID
    assert lib.pi_wait_selftest(FAKE, 1 << 20, 1, 0, None) == pi.PI_ERR_INVALID
    assert lib.pi_wait_selftest(FAKE, 1 << 20, 1, 20000000, None) == pi.PI_ERR_INVALID


@pytest.mark.gpu
@pytest.mark.parametrize("kind", [0, 1])
def test_bounded_wait_runs_out_reports_and_recovers(orc, kind):
    torch = pytest.importorskip("torch")
    from gpu_helpers import TOL, check_mask, device_layer, words_np
    from oracle import rel_l2
    pi = _pi()
    w = synth.WORKLOADS["tiny_relu_512x2048_f32"]
    L, _ = device_layer(w, 0)
    ws = pi.workspace([L], 1)
    assert pi.pi_get_device_status(ws, clear=True)[0] == pi.PI_OK
    t0 = time.perf_counter()
    pi.pi_wait_selftest(ws, kind, 2000)  # 2 ms limit
    st, word = pi.pi_get_device_status(ws, clear=True)
    assert st == pi.PI_ERR_TIMEOUT and word & 4, (st, word)
    assert time.perf_counter() - t0 < 5.0
    assert pi.pi_get_device_status(ws)[0] == pi.PI_OK  # cleared
    # the context and the workspace still work: one fused stack step
    x0 = synth.x_host(w, 0, 1)
    x = torch.from_numpy(x0).cuda()
    tr = torch.zeros((1, 1, (w.d_ff + 31) // 32), dtype=torch.int32, device="cuda")
    pi.pi_ffn_stack([L], x, w.tau, pi.PI_MASK_UNION, mask_trace=tr, ws=ws)
    assert pi.pi_get_device_status(ws)[0] == pi.PI_OK
    xo, _, z = orc.layer_forward(synth.layer_host(w, 0), x0[0], w.tau)
    if check_mask(words_np(tr)[0, 0], z, w.d_ff, w.hot, synth.threshold_logit(w.tau)) == 0:
        assert rel_l2(x.cpu().numpy()[0] - x0[0], xo - x0[0]) <= TOL["f32"]
    assert np.all(np.isfinite(x.cpu().numpy()))
