"""CUDA path vs the CPU oracle at sizes the oracle finishes in seconds, that
span several tiles and have ragged tails: each C-ABI entry point is fed the
oracle's own inputs (masks, lists) and compared element by element.

  masks  : exact outside the 1e-4 threshold band
  lists  : bit-exact (ids and counts)
  FFN y  : relative L2 <= 5e-3 (fp16 / Q4_0 weights), <= 1e-5 (fp32 weights)
"""
import math

import numpy as np
import pytest

from activation_sparse_predictor_b200 import synth
from gpu_helpers import BAND, TOL, check_mask, device_layer, pi_mod, unpack_bits, words_np
from helpers import small_workload
from oracle import rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHAPES = [  # d, F, r, H   (F ragged; H not always a multiple of 32)
    (64, 100, 16, 0),
    (256, 1000, 64, 200),
    (1024, 3001, 128, 640),
]
KINDS = [(act, wdt) for act in ("relu", "reglu", "relu2") for wdt in ("f32", "f16", "q4_0")]


def _wl(act, wdt, shape, seed=41, mean=0.2):
    d, F, r, H = shape
    return small_workload(act, wdt, "f32" if wdt == "f32" else "f16", d=d, F=F, r=r, hot=H,
                          seed=seed, mean=mean)


def _xh(d, batch, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((batch, d))
    return (x / np.sqrt((x * x).mean(axis=1, keepdims=True))).astype(np.float32)


@pytest.fixture(scope="module")
def pi():
    return pi_mod()


# ------------------------------------------------------------------ synth

def test_device_generator_matches_host():
    for wdt in ("f32", "f16", "q4_0"):
        k = synth.key(9, 3, 1)
        h = synth.fill_host(k, 0.03, (37, 256), wdt)
        d = synth.fill_device(k, 0.03, (37, 256), wdt, "cuda")
        torch.cuda.synchronize()
        if wdt == "q4_0":
            assert np.array_equal(h[0], d[0].cpu().numpy())
            assert np.array_equal(h[1], d[1].cpu().numpy().view(np.uint16))
        elif wdt == "f16":
            assert np.array_equal(h.view(np.uint16), d.cpu().numpy().view(np.uint16))
        else:
            assert np.array_equal(h, d.cpu().numpy())


# -------------------------------------------------------------- predictor

@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("pdt", ["f32", "f16"])
@pytest.mark.parametrize("batch", [1, 5, 64])
def test_predict(pi, orc, shape, pdt, batch):
    w = _wl("relu", "f32" if pdt == "f32" else "f16", shape)
    L, _ = device_layer(w, 0)
    H = synth.layer_host(w, 0)
    xh = _xh(w.d_model, batch, 1)
    mask = pi.pi_predict(L, torch.from_numpy(xh).cuda(), 0.5)
    m = words_np(mask)
    for b in range(batch):
        _, z = orc.predict(H, xh[b].astype(np.float64))
        check_mask(m[b], z, w.d_ff, w.hot, 0.0)


def test_predict_threshold(pi, orc):
    """tau != 0.5: the logit threshold moves the mask the same way on both sides."""
    w = _wl("relu", "f16", SHAPES[1])
    L, _ = device_layer(w, 0)
    H = synth.layer_host(w, 0)
    xh = _xh(w.d_model, 2, 2)
    for tau in (0.2, 0.8):
        m = words_np(pi.pi_predict(L, torch.from_numpy(xh).cuda(), tau))
        theta = synth.threshold_logit(tau)
        for b in range(2):
            _, z = orc.predict(H, xh[b].astype(np.float64))
            check_mask(m[b], z, w.d_ff, w.hot, theta)


# -------------------------------------------------------------- compaction

@pytest.mark.parametrize("F", [1, 31, 33, 1000, 32768 + 17, 49152])
@pytest.mark.parametrize("batch", [1, 4, 64])
@pytest.mark.parametrize("density", [0.0, 0.03, 0.5, 1.0])
def test_compact(pi, orc, F, batch, density):
    rng = np.random.default_rng(F * 7 + batch)
    words = (F + 31) // 32
    bits = rng.random((batch, words * 32)) < density
    bits[:, F:] = False
    masks = np.packbits(bits, axis=1, bitorder="little").view(np.uint32).copy()
    dm = torch.from_numpy(masks.view(np.int32)).cuda()
    for begin in sorted({0, min(F, 5), F // 3, F}):
        idx, cnt = pi.pi_compact(dm, F, begin, pi.PI_MASK_UNION)
        want = orc.compact(masks, F, begin)
        n = int(cnt.cpu()[0])
        assert n == len(want)
        assert np.array_equal(idx.cpu().numpy()[0, :n], want)
        idx, cnt = pi.pi_compact(dm, F, begin, pi.PI_MASK_PER_TOKEN)
        ic, cc = idx.cpu().numpy(), cnt.cpu().numpy()
        for b in range(batch):
            want = orc.compact(masks[b], F, begin)
            assert cc[b] == len(want)
            assert np.array_equal(ic[b, :cc[b]], want)


# --------------------------------------------------------------- sparse FFN

def _oracle_masks(orc, H, w, xh):
    ms, zs = [], []
    for b in range(xh.shape[0]):
        _, z = orc.predict(H, xh[b].astype(np.float64))
        ms.append(orc.mask(z, w.d_ff, w.hot, 0.0))
        zs.append(z)
    return np.stack(ms), zs


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("act,wdt", KINDS)
@pytest.mark.parametrize("batch,mode,packed", [(1, "union", False), (3, "per_token", True),
                                               (16, "per_token", False), (64, "union", True),
                                               (5, "union", False), (1, "union", True)])
def test_sparse_ffn(pi, orc, shape, act, wdt, batch, mode, packed):
    w = _wl(act, wdt, shape)
    L, _ = device_layer(w, 0, packed=packed)
    H = synth.layer_host(w, 0)
    xh = _xh(w.d_model, batch, 3)
    masks, _ = _oracle_masks(orc, H, w, xh)
    union = orc.compact(masks, w.d_ff, w.hot)
    m = pi.MODES[mode]
    dev_idx = torch.zeros(max(w.d_ff, 1), dtype=torch.int32, device="cuda")
    dev_idx[: len(union)] = torch.from_numpy(union).cuda()
    dev_cnt = torch.tensor([len(union)], dtype=torch.int32, device="cuda")
    y = pi.pi_sparse_ffn(L, torch.from_numpy(xh).cuda(), torch.from_numpy(masks.view(np.int32)).cuda(),
                         dev_idx, dev_cnt, m).cpu().numpy()
    for b in range(batch):
        own = orc.compact(masks[b], w.d_ff, w.hot) if (mode == "per_token" or batch == 1) else union
        ref = orc.sparse_ffn(H, xh[b].astype(np.float64), own)
        err = rel_l2(y[b], ref)
        assert err <= TOL[wdt], (b, err)


@pytest.mark.parametrize("act", ["relu", "reglu", "relu2"])
@pytest.mark.parametrize("batch,mode", [(3, "per_token"), (5, "union"), (8, "per_token")])
def test_sparse_ffn_cuda_cores_fp16(pi, orc, act, batch, mode, monkeypatch):
    """fp16 layers at 2-15 tokens take the tensor cores; the CUDA-core
    kernels (the path when those are unavailable) still match the oracle."""
    monkeypatch.setenv("PI_DISABLE_TC", "1")
    test_sparse_ffn(pi, orc, (1024, 3001, 128, 640), act, "f16", batch, mode, batch % 2 == 0)


@pytest.mark.parametrize("act,wdt", KINDS)
def test_sparse_ffn_edges(pi, orc, act, wdt):
    """Empty set (y == 0 exactly), everything cold listed, everything hot."""
    d, F, r = 256, 1000, 64
    xh = _xh(d, 2, 4)
    for hot, lst in [(0, np.zeros(0, np.int32)), (0, np.arange(F, dtype=np.int32)),
                     (F, np.zeros(0, np.int32)), (100, np.arange(100, F, 3, dtype=np.int32))]:
        w = _wl(act, wdt, (d, F, r, hot))
        L, _ = device_layer(w, 0)
        H = synth.layer_host(w, 0)
        di = torch.zeros(F, dtype=torch.int32, device="cuda")
        di[: len(lst)] = torch.from_numpy(lst).cuda()
        dc = torch.tensor([len(lst)], dtype=torch.int32, device="cuda")
        y = pi.pi_sparse_ffn(L, torch.from_numpy(xh).cuda(), None, di, dc,
                             pi.PI_MASK_UNION).cpu().numpy()
        for b in range(2):
            ref = orc.sparse_ffn(H, xh[b].astype(np.float64), lst)
            if np.linalg.norm(ref) == 0.0:
                assert np.all(y[b] == 0.0)
            else:
                assert rel_l2(y[b], ref) <= TOL[wdt]


def test_sparse_ffn_is_deterministic(pi):
    w = _wl("reglu", "q4_0", SHAPES[2])
    L, _ = device_layer(w, 0)
    xh = torch.from_numpy(_xh(w.d_model, 1, 5)).cuda()
    lst = torch.arange(w.hot, w.d_ff, 2, dtype=torch.int32, device="cuda")
    cnt = torch.tensor([lst.numel()], dtype=torch.int32, device="cuda")
    ys = [pi.pi_sparse_ffn(L, xh, None, lst, cnt, pi.PI_MASK_UNION).clone() for _ in range(3)]
    assert all(torch.equal(ys[0], v) for v in ys[1:])


def test_device_checks_flag_bad_lists(pi, orc):
    """Out-of-range ids and counts are skipped / clamped and reported."""
    w = _wl("relu", "f16", SHAPES[1])
    L, _ = device_layer(w, 0)
    H = synth.layer_host(w, 0)
    xh = _xh(w.d_model, 1, 6)
    ws = pi.workspace([L], 1)
    good = np.array([300, 301, 999], np.int32)
    bad = np.array([300, 301, 5000, 999], np.int32)
    di = torch.from_numpy(bad).cuda()
    dc = torch.tensor([4], dtype=torch.int32, device="cuda")
    y = pi.pi_sparse_ffn(L, torch.from_numpy(xh).cuda(), None, di, dc, pi.PI_MASK_UNION, ws=ws)
    st, word = pi.pi_get_device_status(ws, clear=True)
    assert st == pi.PI_ERR_DEVICE_CHECK and word & 1
    ref = orc.sparse_ffn(H, xh[0].astype(np.float64), good)
    assert rel_l2(y.cpu().numpy()[0], ref) <= 5e-3
    st, word = pi.pi_get_device_status(ws)
    assert st == pi.PI_OK and word == 0
    dc.fill_(w.d_ff)  # longer than the cold range
    pi.pi_sparse_ffn(L, torch.from_numpy(xh).cuda(), None, di, dc, pi.PI_MASK_UNION, ws=ws)
    st, word = pi.pi_get_device_status(ws, clear=True)
    assert st == pi.PI_ERR_DEVICE_CHECK and word & 2


# -------------------------------------------------------------------- stack

@pytest.mark.parametrize("act,wdt", [("relu", "f32"), ("reglu", "f16"), ("reglu", "q4_0"),
                                     ("relu", "q4_0"), ("relu", "f16"), ("relu2", "f16"),
                                     ("relu2", "q4_0"), ("reglu", "f32")])
@pytest.mark.parametrize("batch,mode", [(1, "union"), (2, "per_token"), (4, "per_token"),
                                        (8, "per_token"), (8, "union")])
@pytest.mark.parametrize("packed", [False, True])
def test_stack(pi, orc, act, wdt, batch, mode, packed):
    """Stacks of 3 layers against the oracle, layer by layer.  The oracle
    runs each layer on the GPU's own masks (from the mask trace), so the
    final x checks the FFN arithmetic of the whole chain; each GPU mask is
    checked against the oracle's logits, exactly outside the 1e-4 band in
    the first layer (same inputs) and outside a band scaled to the path's
    tolerance in later layers, whose inputs differ by the earlier layers'
    rounding (fp16 operands on the tensor cores from 2 tokens on)."""
    w = _wl(act, wdt, (512, 1500, 64, 256), seed=43, mean=0.15).scaled(3)
    dev = [device_layer(w, l, packed=packed) for l in range(w.n_layers)]
    host = [synth.layer_host(w, l) for l in range(w.n_layers)]
    x0 = synth.x_host(w, 0, batch)
    x = torch.from_numpy(x0).cuda()
    words = (w.d_ff + 31) // 32
    trace = torch.zeros((w.n_layers, batch, words), dtype=torch.int32, device="cuda")
    pi.pi_ffn_stack([L for L, _ in dev], x, 0.5, pi.MODES[mode], mask_trace=trace)
    xg = x.cpu().numpy()
    tr = trace.cpu().numpy().view(np.uint32)
    union = mode == "union" and batch > 1
    xs = x0.astype(np.float64)
    for l, H in enumerate(host):
        band = BAND if l == 0 else max(BAND, 4 * TOL[wdt])
        xh = [orc.rmsnorm(xs[b].astype(np.float32)) for b in range(batch)]
        for b in range(batch):
            _, z = orc.predict(H, xh[b])
            check_mask(tr[l, b], z, w.d_ff, w.hot, 0.0, band)
        lists = [orc.compact(tr[l] if union else tr[l, b], w.d_ff, w.hot) for b in range(batch)]
        xs = np.stack([xs[b].astype(np.float32).astype(np.float64) +
                       orc.sparse_ffn(H, xh[b], lists[b]) for b in range(batch)])
    for b in range(batch):
        assert rel_l2(xg[b] - x0[b], xs[b] - x0[b]) <= TOL[wdt], b


@pytest.mark.parametrize("packed", [False, True])
def test_stack_is_deterministic(pi, packed):
    w = _wl("reglu", "q4_0", (512, 1500, 64, 256), seed=44).scaled(4)
    layers = [device_layer(w, l, packed=packed)[0] for l in range(4)]
    x0 = torch.from_numpy(synth.x_host(w, 0, 1)).cuda()
    outs = []
    for _ in range(2):
        x = x0.clone()
        pi.pi_ffn_stack(layers, x, 0.5, pi.PI_MASK_UNION)
        outs.append(x)
    assert torch.equal(outs[0], outs[1])


def test_kernel_launch_counter(pi):
    """One fused launch per batch-1 stack call of at most 40 layers; the same
    count on every repeat of a multi-kernel (batch 4, union) call."""
    w = _wl("reglu", "q4_0", (512, 1500, 64, 256), seed=44).scaled(4)
    layers = [device_layer(w, l, packed=True)[0] for l in range(4)]
    x = torch.from_numpy(synth.x_host(w, 0, 1)).cuda()
    n0 = pi.pi_kernel_launches()
    pi.pi_ffn_stack(layers, x, 0.5, pi.PI_MASK_UNION)
    assert pi.pi_kernel_launches() - n0 == 1
    xb = torch.from_numpy(synth.x_host(w, 0, 4)).cuda()
    counts = []
    for _ in range(2):
        n0 = pi.pi_kernel_launches()
        pi.pi_ffn_stack(layers, xb, 0.5, pi.PI_MASK_UNION)
        counts.append(pi.pi_kernel_launches() - n0)
    assert counts[0] == counts[1] >= 4 * 6  # per layer: norm, predictor, compaction, FFN, reduce


@pytest.mark.parametrize("act", ["reglu", "relu2"])
@pytest.mark.parametrize("batch", [2, 4])
def test_q4_per_token_stack_is_one_fused_pass_per_token(pi, act, batch):
    """A Q4_0 stack at several tokens with per-token masks (no mask trace) runs
    one persistent single-token pass per token: one launch per token, and
    every token's result bit-identical to a batch-1 call on it (the batched
    kernels, taken when a mask trace is asked for, are checked against the
    oracle by test_stack)."""
    w = _wl(act, "q4_0", (512, 1500, 64, 256), seed=45, mean=0.15).scaled(4)
    layers = [device_layer(w, l, packed=True)[0] for l in range(4)]
    x0 = torch.from_numpy(synth.x_host(w, 0, batch)).cuda()
    x = x0.clone()
    n0 = pi.pi_kernel_launches()
    pi.pi_ffn_stack(layers, x, 0.5, pi.PI_MASK_PER_TOKEN)
    assert pi.pi_kernel_launches() - n0 == batch
    for b in range(batch):
        xb = x0[b:b + 1].clone()
        pi.pi_ffn_stack(layers, xb, 0.5, pi.PI_MASK_PER_TOKEN)
        assert torch.equal(xb[0], x[b]), b


@pytest.mark.parametrize("shape", [(1024, 3001, 128, 640), (256, 1000, 64, 200), (512, 2048, 64, 0),
                                   (4096, 1500, 64, 256), (8192, 1000, 64, 640)])
@pytest.mark.parametrize("act", ["relu", "reglu", "relu2"])
@pytest.mark.parametrize("batch,mode", [(2, "per_token"), (5, "union"), (16, "per_token"),
                                        (20, "union"), (48, "per_token"), (64, "union")])
@pytest.mark.parametrize("wdt", ["f16", "q4_0"])
def test_ffn_on_tensor_cores(pi, orc, shape, act, batch, mode, wdt, monkeypatch):
    """At 2-64 tokens an fp16 layer's listed rows (hot prefix and cold list;
    whole-hot tiles loaded as boxes, the others gathered four rows per TMA
    load) run on the tensor cores (fp16 inputs, fp32 accumulation): within
    the fp16 tolerance of the oracle, close to the CUDA-core path, and not
    bitwise equal to it (so the tensor-core path did run).  Shapes cover a
    ragged d_ff, a hot prefix that ends inside a tile, and no hot prefix;
    batches 2, 5, 20 and 48 pad the token tile.  At d = 4096 and 8192 the up
    kernel splits d over 2 and 4 CTAs per row tile, and the down kernel
    splits a short list over 8 and 4 CTAs per column tile.  Q4_0 layers take
    the same path with their rows decoded to fp16 in shared memory (within
    the Q4_0 tolerance; 4e-3 of the CUDA-core path, which decodes to fp32)."""
    w = _wl(act, wdt, shape, seed=47)
    L, _ = device_layer(w, 0, packed=(batch % 32 == 0))
    H = synth.layer_host(w, 0)
    xh = _xh(w.d_model, batch, 9)
    masks, _ = _oracle_masks(orc, H, w, xh)
    union = orc.compact(masks, w.d_ff, w.hot)
    dev_idx = torch.zeros(w.d_ff, dtype=torch.int32, device="cuda")
    dev_idx[: len(union)] = torch.from_numpy(union).cuda()
    dev_cnt = torch.tensor([len(union)], dtype=torch.int32, device="cuda")
    dxh = torch.from_numpy(xh).cuda()
    dmask = torch.from_numpy(masks.view(np.int32)).cuda()
    m = pi.MODES[mode]

    def run():
        return pi.pi_sparse_ffn(L, dxh, dmask, dev_idx, dev_cnt, m).cpu().numpy()

    y_tc = run()
    monkeypatch.setenv("PI_DISABLE_TC", "1")
    y_cc = run()
    monkeypatch.delenv("PI_DISABLE_TC")
    assert not np.array_equal(y_tc, y_cc)
    for b in range(batch):
        own = orc.compact(masks[b], w.d_ff, w.hot) if mode == "per_token" else union
        ref = orc.sparse_ffn(H, xh[b].astype(np.float64), own)
        if np.linalg.norm(ref) == 0.0:
            assert np.all(y_tc[b] == 0.0)
            continue
        assert rel_l2(y_tc[b], ref) <= TOL[wdt], b
        assert rel_l2(y_tc[b], y_cc[b]) <= (2e-3 if wdt == "f16" else 4e-3), b
    assert np.array_equal(run(), y_tc)  # deterministic


@pytest.mark.parametrize("shape", [(1024, 3001, 256, 640), (512, 2048, 128, 200)])
@pytest.mark.parametrize("batch", [2, 7, 16, 20, 64])
@pytest.mark.parametrize("tau", [0.5, 0.3])
def test_predict_on_tensor_cores(pi, orc, shape, batch, tau, monkeypatch):
    """At 2-64 tokens the fp16 predictor runs on the tensor cores with the
    fp32 vectors split into fp16 hi + lo parts: masks equal the oracle's
    outside the 1e-4 band (hot bits set, tail bits clear), including a hot
    prefix that ends inside a mask word, and equal the CUDA-core path's
    outside the band."""
    w = _wl("relu", "f16", shape, seed=53)
    L, _ = device_layer(w, 0)
    H = synth.layer_host(w, 0)
    xh = _xh(w.d_model, batch, 5)
    dxh = torch.from_numpy(xh).cuda()
    m_tc = words_np(pi.pi_predict(L, dxh, tau))
    monkeypatch.setenv("PI_DISABLE_TC", "1")
    m_cc = words_np(pi.pi_predict(L, dxh, tau))
    monkeypatch.delenv("PI_DISABLE_TC")
    theta = synth.threshold_logit(tau)
    for b in range(batch):
        _, z = orc.predict(H, xh[b].astype(np.float64))
        check_mask(m_tc[b], z, w.d_ff, w.hot, theta)
        check_mask(m_cc[b], z, w.d_ff, w.hot, theta)
