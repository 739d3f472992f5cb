"""pi_predict_noalloc: the predictor with its hidden vector u in the
library's static per-device buffer instead of a workspace, for callers that
cannot allocate device memory.  Named to be collected last, so it also runs
after every other test in one process."""
import ctypes

import numpy as np
import pytest

from activation_sparse_predictor_b200 import synth

FAKE = 1 << 20  # 256-byte aligned stand-in address: never dereferenced here


def _pi():
    from activation_sparse_predictor_b200 import build
    build.build_libpi()
    from activation_sparse_predictor_b200 import pi
    return pi


def test_noalloc_rejects_batch_times_rank_beyond_its_buffer():
    pi = _pi()
    L = pi.pi_layer(64, 256, 8192, 32, pi.PI_RELU, pi.PI_F16, pi.PI_F16, None, FAKE, FAKE,
                    None, None, None, FAKE, FAKE, FAKE, FAKE)
    # 32 * 8192 = the limit: passes validation up to the buffer check; 33 * 8192 does not
    assert 32 * 8192 == pi.PI_PREDICT_NOALLOC_MAX_FLOATS
    st = pi._lib.pi_predict_noalloc(ctypes.byref(L), FAKE, 33, 0.5, FAKE, None)
    assert pi.pi_status_string(st) == "PI_ERR_INVALID"
    assert "static scratch" in pi.pi_last_error()


@pytest.mark.gpu
def test_noalloc_matches_predict_on_consecutive_calls():
    """One token (both entry points on the CUDA-core kernels): bit-identical
    masks on two calls in a row, each on a fresh input."""
    torch = pytest.importorskip("torch")
    from gpu_helpers import device_layer, words_np
    pi = _pi()
    w = synth.WORKLOADS["relullama7b_reglu_4096x11008_f16"]
    L, _ = device_layer(w, 0)
    batch = 1
    words = (w.d_ff + 31) // 32
    for call in range(2):
        xh = synth.x_device(w, 10 + call, batch)
        want = pi.pi_predict(L, xh, w.tau)
        got = torch.full((batch, words), -1, dtype=torch.int32, device="cuda")
        pi.pi_predict_noalloc(L, xh, w.tau, got)
        torch.cuda.synchronize()
        assert np.array_equal(words_np(got), words_np(want)), call


@pytest.mark.gpu
@pytest.mark.parametrize("batch", [4, 16, 64])
def test_noalloc_matches_oracle_at_token_batches(orc, batch):
    """At 4, 16 and 64 tokens pi_predict runs the tensor-core predictor and
    pi_predict_noalloc the CUDA-core one: both must match the oracle's mask
    outside the 1e-4 logit band, so they agree there too; two calls in a row."""
    torch = pytest.importorskip("torch")
    from gpu_helpers import BAND, check_mask, device_layer, unpack_bits, words_np
    pi = _pi()
    w = synth.WORKLOADS["relullama7b_reglu_4096x11008_f16"]
    L, _ = device_layer(w, 0)
    H = synth.layer_host(w, 0)
    words = (w.d_ff + 31) // 32
    theta = synth.threshold_logit(w.tau)
    for call in range(2):
        x = synth.x_host(w, 20 + call, batch)
        xh = torch.from_numpy(x).cuda()
        got = torch.full((batch, words), -1, dtype=torch.int32, device="cuda")
        pi.pi_predict_noalloc(L, xh, w.tau, got)
        want = pi.pi_predict(L, xh, w.tau)
        torch.cuda.synchronize()
        g, t = words_np(got), words_np(want)
        for b in range(0, batch, 5 if batch > 16 else 1):
            _, z = orc.predict(H, x[b].astype(np.float64))
            check_mask(g[b], z, w.d_ff, w.hot, theta)
            check_mask(t[b], z, w.d_ff, w.hot, theta)
            outside = np.abs(z - theta) > BAND
            gb, _ = unpack_bits(g[b], w.d_ff)
            tb, _ = unpack_bits(t[b], w.d_ff)
            assert np.array_equal(gb[outside], tb[outside]), (call, b)
