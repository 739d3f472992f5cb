"""CUDA path vs the CPU oracle at the five workloads' full layer shapes, in
the launch configuration the benchmark times (pi_ffn_stack), plus the
headline 80-layer Llama2-70B-shaped Q4_0 stack.  Where the oracle would be
too slow (64-token union batches) it checks a sample of tokens one by one;
masks of every token are checked."""
import numpy as np
import pytest

from activation_sparse_predictor_b200 import synth
from gpu_helpers import TOL, check_mask, device_layer, pi_mod, words_np
from oracle import rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

NAMES = synth.WORKLOAD_ORDER


@pytest.fixture(scope="module")
def pi():
    return pi_mod()


def _run_layer_stack(pi, L, x0, mode, words):
    batch = x0.shape[0]
    x = torch.from_numpy(x0).cuda()
    trace = torch.zeros((1, batch, words), dtype=torch.int32, device="cuda")
    pi.pi_ffn_stack([L], x, 0.5, mode, mask_trace=trace)
    return x.cpu().numpy(), words_np(trace)[0]


@pytest.mark.parametrize("name", NAMES)
def test_workload_layer_decode(pi, orc, name):
    w = synth.WORKLOADS[name]
    layer = w.n_layers - 1
    L, _ = device_layer(w, layer, packed=True)
    H = synth.layer_host(w, layer)
    words = (w.d_ff + 31) // 32
    for batch in w.batches:
        x0 = synth.x_host(w, 0, batch)
        xg, tr = _run_layer_stack(pi, L, x0, pi.PI_MASK_PER_TOKEN, words)
        flips = 0
        for b in range(batch):
            xo, m, z = orc.layer_forward(H, x0[b], w.tau)
            f = check_mask(tr[b], z, w.d_ff, w.hot, synth.threshold_logit(w.tau))
            flips += f
            if f:
                # a band neuron decided differently: compare over the GPU's own
                # neuron set (teacher-forced mask) instead of skipping the token
                xhb = orc.rmsnorm(x0[b])
                xo = x0[b] + orc.sparse_ffn(H, xhb, orc.compact(tr[b], w.d_ff, w.hot))
            assert rel_l2(xg[b] - x0[b], xo - x0[b]) <= TOL[w.w_dtype], (name, batch, b)
        assert flips <= max(1, batch // 4), f"{flips} band flips over {batch} tokens"
        # the separate entry points on the oracle's own mask
        xh = np.stack([orc.rmsnorm(x0[b]) for b in range(batch)]).astype(np.float32)
        _, z0 = orc.predict(H, xh[0].astype(np.float64))
        m0 = orc.mask(z0, w.d_ff, w.hot, 0.0)
        dm = torch.from_numpy(m0.view(np.int32)[None]).cuda()
        idx, cnt = pi.pi_compact(dm, w.d_ff, w.hot, pi.PI_MASK_UNION)
        lst = orc.compact(m0, w.d_ff, w.hot)
        assert int(cnt.cpu()[0]) == len(lst)
        assert np.array_equal(idx.cpu().numpy()[0, :len(lst)], lst)
        y = pi.pi_sparse_ffn(L, torch.from_numpy(xh[:1]).cuda(), None, idx, cnt,
                             pi.PI_MASK_UNION).cpu().numpy()[0]
        assert rel_l2(y, orc.sparse_ffn(H, xh[0].astype(np.float64), lst)) <= TOL[w.w_dtype]


@pytest.mark.parametrize("name", [n for n in NAMES if synth.WORKLOADS[n].union_batches])
def test_workload_layer_union(pi, orc, name):
    w = synth.WORKLOADS[name]
    L, _ = device_layer(w, 0, packed=True)
    H = synth.layer_host(w, 0)
    words = (w.d_ff + 31) // 32
    for batch in w.union_batches:
        x0 = synth.x_host(w, 1, batch)
        xg, tr = _run_layer_stack(pi, L, x0, pi.PI_MASK_UNION, words)
        xh = []
        for b in range(batch):
            xhb = orc.rmsnorm(x0[b])
            _, z = orc.predict(H, xhb)
            check_mask(tr[b], z, w.d_ff, w.hot, 0.0)  # exact outside the band
            xh.append(xhb)
        # teacher-forced: the FFN over the union of the masks the GPU decided
        # (they differ from the oracle's only inside the band)
        union = orc.compact(tr.copy(), w.d_ff, w.hot)
        for b in (0, batch // 2 + 5, batch - 1):
            ref = orc.sparse_ffn(H, xh[b], union)
            assert rel_l2(xg[b] - x0[b], ref) <= TOL[w.w_dtype], (name, b)


def test_headline_stack_80_layers(pi, orc):
    """Llama2-70B-shaped Q4_0 ReGLU stack, 80 layers, batch 1: masks of the
    first layers match the oracle chain, a 2-layer chain matches end to end,
    and the whole stack is bitwise reproducible."""
    w = synth.WORKLOADS["llama2_70b_reglu_8192x28672_q4_0"]
    layers = [device_layer(w, l, packed=True)[0] for l in range(w.n_layers)]
    words = (w.d_ff + 31) // 32
    x0 = synth.x_host(w, 0, 1)
    outs, trace = [], None
    for rep in range(2):
        x = torch.from_numpy(x0).cuda()
        tr = torch.zeros((w.n_layers, 1, words), dtype=torch.int32, device="cuda")
        pi.pi_ffn_stack(layers, x, 0.5, pi.PI_MASK_UNION, mask_trace=tr)
        outs.append(x.cpu().numpy())
        trace = words_np(tr)
    assert np.array_equal(outs[0], outs[1])
    assert np.all(np.isfinite(outs[0]))
    # oracle chain over the first two layers
    xr = x0[0].astype(np.float64)
    for l in range(2):
        H = synth.layer_host(w, l)
        xo, m, z = orc.layer_forward(H, xr.astype(np.float32), 0.5)
        assert check_mask(trace[l, 0], z, w.d_ff, w.hot, 0.0) == 0
        xr = xo
    x = torch.from_numpy(x0).cuda()
    pi.pi_ffn_stack(layers[:2], x, 0.5, pi.PI_MASK_UNION)
    assert rel_l2(x.cpu().numpy()[0] - x0[0], xr - x0[0]) <= TOL["q4_0"]


def test_tiny_workload_all_16_vectors(pi, orc):
    """The tiny ReLU workload states 16 input vectors: every one through the
    benchmarked single-token path, against the oracle."""
    w = synth.WORKLOADS["tiny_relu_512x2048_f32"]
    L, _ = device_layer(w, 0, packed=True)
    H = synth.layer_host(w, 0)
    words = (w.d_ff + 31) // 32
    assert w.steps == 16
    for step in range(w.steps):
        x0 = synth.x_host(w, step, 1)
        xg, tr = _run_layer_stack(pi, L, x0, pi.PI_MASK_UNION, words)
        xo, m, z = orc.layer_forward(H, x0[0], w.tau)
        if check_mask(tr[0], z, w.d_ff, w.hot, 0.0):
            xo = x0[0] + orc.sparse_ffn(H, orc.rmsnorm(x0[0]), orc.compact(tr[0], w.d_ff, w.hot))
        assert rel_l2(xg[0] - x0[0], xo - x0[0]) <= TOL["f32"], step


def test_relullama_256_decode_steps(pi, orc):
    """The ReluLLaMA-7B-shaped workload states 256 decode steps: each step's
    token through its first layer on the benchmarked single-token path, mask
    and output against the oracle (teacher-forced mask where a band neuron
    flipped)."""
    w = synth.WORKLOADS["relullama7b_reglu_4096x11008_f16"]
    L, _ = device_layer(w, 0, packed=True)
    H = synth.layer_host(w, 0)
    words = (w.d_ff + 31) // 32
    assert w.steps == 256
    flips = 0
    ws = pi.workspace([L], 1)
    for step in range(w.steps):
        x0 = synth.x_host(w, step, 1)
        x = torch.from_numpy(x0).cuda()
        tr = torch.zeros((1, 1, words), dtype=torch.int32, device="cuda")
        pi.pi_ffn_stack([L], x, w.tau, pi.PI_MASK_UNION, mask_trace=tr, ws=ws)
        xg, t = x.cpu().numpy()[0], words_np(tr)[0, 0]
        xo, m, z = orc.layer_forward(H, x0[0], w.tau)
        f = check_mask(t, z, w.d_ff, w.hot, 0.0)
        flips += f
        if f:
            xo = x0[0] + orc.sparse_ffn(H, orc.rmsnorm(x0[0]), orc.compact(t, w.d_ff, w.hot))
        assert rel_l2(xg - x0[0], xo - x0[0]) <= TOL["f16"], step
    assert flips <= 8, f"{flips} band flips over 256 steps"
    st, word = pi.pi_get_device_status(ws)
    assert st == pi.PI_OK, hex(word)
