"""The benchmarked batch-1 path end to end: stacks deeper than one launch of
the persistent kernel (it runs at most 40 layers per launch), checked layer
by layer against the oracle, so the hand-off of x, of the mask trace and of
the layer pointers at the launch boundaries (layers 40 and 80) is pinned.

For every prefix length n the stack is run from the same x0 on the GPU; by
determinism the prefix's output is the full stack's x after n layers (this
is asserted for the whole stack).  Layer n-1 is then checked teacher-forced
(same input x, same mask; the pages' reading of stack parity):
  * its traced mask equals the oracle's outside the 1e-4 logit band;
  * its cold list (pi_read_list) equals the oracle's compaction of that
    mask, bit for bit;
  * the listed-row counter equals hot + that list's length exactly, and the
    down-row counter lies within the rows the oracle's first-matrix
    pre-activations put surely above zero and those near zero;
  * x_n - x_{n-1} matches the oracle's FFN output over the same neuron set
    at relative L2 <= the dtype's tolerance.
"""
import numpy as np
import pytest

from activation_sparse_predictor_b200 import synth
from gpu_helpers import TOL, check_mask, device_layer, pi_mod, words_np
from helpers import np_decode
from oracle import rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

N_LAYERS = 84  # crosses the persistent kernel's launch boundaries at 40 and 80


def _workload(act, w_dtype, seed):
    return synth.Workload(
        name=f"chain_{act}_512x1500_{w_dtype}", act=act, d_model=512, d_ff=1500, rank=64,
        n_layers=N_LAYERS, hot=256, w_dtype=w_dtype, p_dtype="f16" if w_dtype != "f32" else "f32",
        seed=seed, tau=0.5, p_rule=("mean", 0.15, 1.0), steps=1)


CASES = [("reglu", "q4_0", 31), ("relu", "f16", 32), ("reglu", "f16", 33), ("relu", "f32", 34),
         ("relu2", "q4_0", 35)]


def _first_preact(H, xh):
    """First-matrix pre-activation (gate for ReGLU, up for ReLU) + bias, in
    float64 from numpy's own decode: decides which down rows are read."""
    w = H["workload"]
    W = np_decode(H["w_gate"] if w.act == "reglu" else H["w_up"], w.w_dtype)  # relu2: up
    return W @ xh + np.asarray(H["bias"], np.float64)


@pytest.mark.parametrize("act,w_dtype,seed", CASES)
def test_stack_prefixes_cross_launch_boundaries(orc, act, w_dtype, seed):
    pi = pi_mod()
    w = _workload(act, w_dtype, seed)
    layers = [device_layer(w, l, packed=True)[0] for l in range(N_LAYERS)]
    hosts = [synth.layer_host(w, l) for l in range(N_LAYERS)]
    words = (w.d_ff + 31) // 32
    theta = synth.threshold_logit(w.tau)
    x0 = synth.x_host(w, 0, 1)
    ws = pi.workspace(layers, 1)

    # the whole stack, with its mask trace
    xf = torch.from_numpy(x0).cuda()
    trace = torch.zeros((N_LAYERS, 1, words), dtype=torch.int32, device="cuda")
    pi.pi_ffn_stack(layers, xf, w.tau, pi.PI_MASK_UNION, mask_trace=trace, ws=ws)
    full_trace = words_np(trace)[:, 0]
    st, word = pi.pi_get_device_status(ws)
    assert st == pi.PI_OK, hex(word)

    x_prev = x0[0].copy()
    flips = 0
    prev_listed = prev_down = 0
    for n in range(1, N_LAYERS + 1):
        x = torch.from_numpy(x0).cuda()
        tr = torch.zeros((n, 1, words), dtype=torch.int32, device="cuda")
        pi.pi_read_counters(ws, clear=True)
        pi.pi_ffn_stack(layers[:n], x, w.tau, pi.PI_MASK_UNION, mask_trace=tr, ws=ws)
        lst = pi.pi_read_list(layers[:n], 1, ws)
        listed, down, second = pi.pi_read_counters(ws, clear=True)
        # ReGLU reads W_up rows exactly where it reads down rows (gate > 0)
        assert second == (down if act == "reglu" else 0)
        xn = x.cpu().numpy()[0]
        trn = words_np(tr)[:, 0]
        assert np.array_equal(trn, full_trace[:n]), f"prefix {n}: trace differs from the full run"
        l = n - 1
        H = hosts[l]
        # teacher-forced: the oracle from the GPU's own input to layer l
        xh = orc.rmsnorm(x_prev)
        _, z = orc.predict(H, xh)
        flips += check_mask(trn[l], z, w.d_ff, w.hot, theta)
        want = orc.compact(trn[l], w.d_ff, w.hot)
        assert np.array_equal(lst, want), f"layer {l}: cold list differs from the oracle's"
        # prefix n reads what prefix n-1 read, plus layer l's rows
        assert listed - prev_listed == w.hot + len(want), f"layer {l}: listed-row counter"
        g = _first_preact(H, xh)
        S = np.concatenate([np.arange(w.hot), want])
        sure, near = int((g[S] > 1e-3).sum()), int((np.abs(g[S]) <= 1e-3).sum())
        assert sure <= down - prev_down <= sure + near, f"layer {l}: down rows"
        prev_listed, prev_down = listed, down
        y = orc.sparse_ffn(H, xh, want)
        assert rel_l2(xn - x_prev, y) <= TOL[w.w_dtype], f"layer {l}"
        x_prev = xn
    assert np.array_equal(xn, xf.cpu().numpy()[0]), "prefix run differs from the full stack"
    assert flips <= 2, f"{flips} band neurons flipped over {N_LAYERS} layers"


@pytest.mark.parametrize("act,w_dtype,seed", CASES[:2])
def test_single_layer_row_counters(orc, act, w_dtype, seed):
    """One fused layer: listed rows == hot + list length exactly; down rows
    (rows whose h != 0) within the oracle's sure / near-zero bracket."""
    pi = pi_mod()
    w = _workload(act, w_dtype, seed).scaled(1)
    L, _ = device_layer(w, 0, packed=True)
    H = synth.layer_host(w, 0)
    words = (w.d_ff + 31) // 32
    ws = pi.workspace([L], 1)
    for step in range(4):
        x0 = synth.x_host(w, step, 1)
        x = torch.from_numpy(x0).cuda()
        tr = torch.zeros((1, 1, words), dtype=torch.int32, device="cuda")
        pi.pi_read_counters(ws, clear=True)
        pi.pi_ffn_stack([L], x, w.tau, pi.PI_MASK_UNION, mask_trace=tr, ws=ws)
        listed, down, second = pi.pi_read_counters(ws, clear=True)
        assert second == (down if act == "reglu" else 0)
        lst = orc.compact(words_np(tr)[0, 0], w.d_ff, w.hot)
        assert listed == w.hot + len(lst)
        xh = orc.rmsnorm(x0[0])
        g = _first_preact(H, xh)
        S = np.concatenate([np.arange(w.hot), lst])
        sure, near = int((g[S] > 1e-3).sum()), int((np.abs(g[S]) <= 1e-3).sum())
        assert sure <= down <= sure + near, (step, down, sure, near)
