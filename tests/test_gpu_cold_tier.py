"""Hybrid cold tier: rows [hot, d_ff) of the FFN weights in page-locked host
memory, read by the GPU over the host link and merged with the hot rows in
the same kernels (QbitAI article, §"Гибридный дизайн вывода CPU/GPU": hot
neurons on the GPU, cold neurons in host memory, results merged on the GPU).

The device copies of the cold rows are overwritten with NaN bit patterns
before the cold-tier call, so any read of them shows in the output.  The
result must equal, bit for bit, the same layer with every row in device
memory on the same (CUDA-core) kernels, and match the oracle within the
path's tolerance.
"""
import ctypes

import numpy as np
import pytest

from activation_sparse_predictor_b200 import synth
from gpu_helpers import BAND, TOL, check_mask, device_layer, pi_mod
from helpers import small_workload
from oracle import rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

KINDS = [(act, wdt) for act in ("relu", "reglu", "relu2") for wdt in ("f32", "f16", "q4_0")]


@pytest.fixture(scope="module")
def pi():
    return pi_mod()


def _wl(act, wdt, shape=(512, 1500, 64, 256), seed=47, n_layers=1):
    d, F, r, H = shape
    w = small_workload(act, wdt, "f32" if wdt == "f32" else "f16", d=d, F=F, r=r, hot=H,
                       seed=seed, mean=0.15)
    return w.scaled(n_layers) if n_layers > 1 else w


def _poison_cold_rows(L):
    """NaN bit patterns (all bytes 0xFF) in device rows [hot, d_ff) of every
    weight buffer of L: the cold-tier layer must not read them."""
    seen = set()
    for name in ("w_gate", "w_up", "w_down_t"):
        v = L.tensors.get(name)
        if v is None:
            continue
        for t in (v if isinstance(v, tuple) else (v,)):
            b = t
            while b._base is not None:
                b = b._base
            if b.data_ptr() in seen:
                continue
            seen.add(b.data_ptr())
            rows = b.reshape(L.d_ff, -1)
            rows[L.hot:].view(torch.uint8).fill_(0xFF)


def _list_and_masks(orc, w, H, xh):
    masks = []
    for b in range(xh.shape[0]):
        _, z = orc.predict(H, xh[b].astype(np.float64))
        masks.append(orc.mask(z, w.d_ff, w.hot, 0.0))
    masks = np.stack(masks)
    return masks, orc.compact(masks, w.d_ff, w.hot)


def _xh(d, batch, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((batch, d))
    return (x / np.sqrt((x * x).mean(axis=1, keepdims=True))).astype(np.float32)


@pytest.mark.parametrize("act,wdt", KINDS)
@pytest.mark.parametrize("batch,mode,packed", [(1, "union", False), (1, "union", True),
                                               (3, "per_token", True), (16, "per_token", False),
                                               (20, "union", True), (40, "union", False),
                                               (64, "per_token", True)])
def test_cold_tier_sparse_ffn(pi, orc, act, wdt, batch, mode, packed, monkeypatch):
    monkeypatch.setenv("PI_DISABLE_TC", "1")  # the device-resident run on the same kernels
    w = _wl(act, wdt)
    L, _ = device_layer(w, 0, packed=packed)
    H = synth.layer_host(w, 0)
    xh = _xh(w.d_model, batch, 5)
    masks, union = _list_and_masks(orc, w, H, xh)
    m = pi.MODES[mode]
    idx = torch.zeros(w.d_ff, dtype=torch.int32, device="cuda")
    idx[: len(union)] = torch.from_numpy(union).cuda()
    cnt = torch.tensor([len(union)], dtype=torch.int32, device="cuda")
    xd = torch.from_numpy(xh).cuda()
    md = torch.from_numpy(masks.view(np.int32)).cuda()
    y_dev = pi.pi_sparse_ffn(L, xd, md, idx, cnt, m).clone()
    Lc = L.with_host_cold_tier()
    _poison_cold_rows(L)
    ws = pi.workspace([Lc], batch)
    pi.pi_read_cold_counters(ws, clear=True)
    y = pi.pi_sparse_ffn(Lc, xd, md, idx, cnt, m, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(y, y_dev)
    yn = y.cpu().numpy()
    for b in range(batch):
        own = orc.compact(masks[b], w.d_ff, w.hot) if (mode == "per_token" or batch == 1) else union
        ref = orc.sparse_ffn(H, xh[b].astype(np.float64), own)
        assert rel_l2(yn[b], ref) <= TOL[wdt], b
    listed, down, second = pi.pi_read_cold_counters(ws)
    # each listed cold row crossed the host link once: at token batches of
    # several chunks the up kernel reads them from their device stage
    assert listed == len(union)
    assert second == (len(union) if act == "reglu" else 0)
    if batch == 1:
        # every listed neuron is cold; its first matrix (and ReGLU's W_up) came
        # over the host link, and its down row when its h was nonzero
        assert listed == len(union)
        assert second == (len(union) if act == "reglu" else 0)
        h, _ = orc.ffn(H, xh[0].astype(np.float64), orc.rowset(w.d_ff, w.hot, union))
        nz = int(np.count_nonzero(h[union]))
        assert down <= listed and abs(down - nz) <= max(2, len(union) // 100), (down, nz)
    else:
        # down rows: once per token chunk of <= 8, or once in all when the
        # down kernel takes four chunks or more (then they are staged too)
        chunks = (batch + 7) // 8
        assert down <= (listed if chunks >= 4 else listed * chunks)


@pytest.mark.parametrize("act", ["relu", "reglu", "relu2"])
@pytest.mark.parametrize("batch,mode,packed", [(2, "per_token", True), (5, "union", False),
                                               (16, "per_token", True), (64, "union", True),
                                               (64, "per_token", False)])
def test_cold_tier_q4_on_tensor_cores(pi, orc, act, batch, mode, packed):
    """Q4_0 layers at token batches take the tensor-core kernels with a cold
    tier too: the listed cold rows (and every listed down row) are staged in
    device memory once, then read by the same kernels, so the result equals
    the device-resident layer's bit for bit."""
    w = _wl(act, "q4_0", (1024, 3001, 128, 640), seed=49)
    L, _ = device_layer(w, 0, packed=packed)
    H = synth.layer_host(w, 0)
    xh = _xh(w.d_model, batch, 8)
    masks, union = _list_and_masks(orc, w, H, xh)
    m = pi.MODES[mode]
    idx = torch.zeros(w.d_ff, dtype=torch.int32, device="cuda")
    idx[: len(union)] = torch.from_numpy(union).cuda()
    cnt = torch.tensor([len(union)], dtype=torch.int32, device="cuda")
    xd = torch.from_numpy(xh).cuda()
    md = torch.from_numpy(masks.view(np.int32)).cuda()
    n0 = pi.pi_kernel_launches()
    y_dev = pi.pi_sparse_ffn(L, xd, md, idx, cnt, m).clone()
    launches_dev = pi.pi_kernel_launches() - n0
    Lc = L.with_host_cold_tier()
    _poison_cold_rows(L)
    ws = pi.workspace([Lc], batch)
    pi.pi_read_cold_counters(ws, clear=True)
    pi.pi_read_counters(ws, clear=True)
    n0 = pi.pi_kernel_launches()
    y = pi.pi_sparse_ffn(Lc, xd, md, idx, cnt, m, ws=ws)
    launches = pi.pi_kernel_launches() - n0
    torch.cuda.synchronize()
    assert torch.equal(y, y_dev)
    yn = y.cpu().numpy()
    for b in range(batch):
        own = orc.compact(masks[b], w.d_ff, w.hot) if mode == "per_token" else union
        ref = orc.sparse_ffn(H, xh[b].astype(np.float64), own)
        assert rel_l2(yn[b], ref) <= TOL["q4_0"], b
    listed, down, second = pi.pi_read_cold_counters(ws)
    assert listed == len(union) and down == len(union)
    assert second == (len(union) if act == "reglu" else 0)
    # the tensor-core path read every listed row once (its own counters)
    rows_listed, rows_down, _ = pi.pi_read_counters(ws)
    assert rows_listed == w.hot + len(union) and rows_down == w.hot + len(union)
    assert launches == launches_dev + 2  # the two staging kernels, then the same FFN kernels


@pytest.mark.parametrize("act,wdt", [("reglu", "q4_0"), ("relu", "f16"), ("relu2", "f32")])
@pytest.mark.parametrize("batch,mode", [(1, "union"), (4, "per_token"), (8, "union")])
def test_cold_tier_stack(pi, orc, act, wdt, batch, mode, monkeypatch):
    """A 3-layer stack with every layer's cold rows in host memory, against
    the oracle layer by layer on the GPU's own masks (as the device-resident
    stack test does), and bit for bit against the device-resident stack on
    the same CUDA-core kernels at token batches."""
    monkeypatch.setenv("PI_DISABLE_TC", "1")
    w = _wl(act, wdt, seed=48, n_layers=3)
    dev = [device_layer(w, l, packed=True)[0] for l in range(w.n_layers)]
    host = [synth.layer_host(w, l) for l in range(w.n_layers)]
    x0 = synth.x_host(w, 0, batch)
    words = (w.d_ff + 31) // 32
    ref_x = None
    # the device-resident stack on the same kernels: token batches, except
    # Q4_0 per-token stacks (with the tensor cores off, one fused pass per
    # token there)
    if batch > 1 and not (wdt == "q4_0" and mode == "per_token"):
        xr = torch.from_numpy(x0).cuda()
        pi.pi_ffn_stack(dev, xr, 0.5, pi.MODES[mode])
        ref_x = xr.clone()
    cold = [L.with_host_cold_tier() for L in dev]
    for L in dev:
        _poison_cold_rows(L)
    x = torch.from_numpy(x0).cuda()
    trace = torch.zeros((w.n_layers, batch, words), dtype=torch.int32, device="cuda")
    pi.pi_ffn_stack(cold, x, 0.5, pi.MODES[mode], mask_trace=trace)
    torch.cuda.synchronize()
    if ref_x is not None:
        assert torch.equal(x, ref_x)
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
    assert np.isfinite(xg).all()
    for b in range(batch):
        assert rel_l2(xg[b] - x0[b], xs[b] - x0[b]) <= TOL[wdt], b


def test_cold_tier_edges(pi, orc, monkeypatch):
    """All rows cold (hot = 0), no rows cold (hot = d_ff) and an empty list."""
    monkeypatch.setenv("PI_DISABLE_TC", "1")
    d, F, r = 256, 1000, 64
    xh = torch.from_numpy(_xh(d, 2, 6)).cuda()
    for hot, lst in [(0, np.arange(0, F, 2, dtype=np.int32)), (F, np.zeros(0, np.int32)),
                     (100, np.zeros(0, np.int32))]:
        w = _wl("reglu", "q4_0", (d, F, r, hot))
        L, _ = device_layer(w, 0, packed=True)
        H = synth.layer_host(w, 0)
        di = torch.zeros(F, dtype=torch.int32, device="cuda")
        di[: len(lst)] = torch.from_numpy(lst).cuda()
        dc = torch.tensor([len(lst)], dtype=torch.int32, device="cuda")
        y_dev = pi.pi_sparse_ffn(L, xh, None, di, dc, pi.PI_MASK_UNION).clone()
        Lc = L.with_host_cold_tier() if hot < F else L
        if hot < F:
            _poison_cold_rows(L)
        y = pi.pi_sparse_ffn(Lc, xh, None, di, dc, pi.PI_MASK_UNION)
        assert torch.equal(y, y_dev)
        for b in range(2):
            ref = orc.sparse_ffn(H, xh[b].cpu().numpy().astype(np.float64), lst)
            if np.linalg.norm(ref) == 0.0:
                assert torch.all(y[b] == 0)
            else:
                assert rel_l2(y[b].cpu().numpy(), ref) <= TOL["q4_0"]


def test_cold_tier_rejects_memory_the_device_cannot_read(pi):
    """Cold pointers into device memory, pageable host memory, or an
    incomplete set are rejected before anything is enqueued."""
    w = _wl("reglu", "f16")
    L, _ = device_layer(w, 0)
    x = torch.from_numpy(synth.x_host(w, 0, 1)).cuda()
    x_before = x.clone()
    pageable = np.zeros(w.d_ff * w.d_model * 2 + 64, np.uint8)
    p_host = (pageable.ctypes.data + 15) // 16 * 16
    dev_buf = torch.empty(w.d_ff * w.d_model * 2, dtype=torch.uint8, device="cuda")
    for fill in (dev_buf.data_ptr(), p_host):
        c = pi.pi_layer()
        ctypes.pointer(c)[0] = L.c
        c.w_gate_cold = c.w_up_cold = c.w_down_t_cold = fill
        bad = pi.Layer.__new__(pi.Layer)
        bad.__dict__.update(L.__dict__)
        bad.c = c
        with pytest.raises(pi.PiError) as e:
            pi.pi_ffn_stack([bad], x, 0.5, pi.PI_MASK_UNION)
        assert e.value.status == pi.PI_ERR_INVALID and "page-locked" in str(e.value)
    Lc = L.with_host_cold_tier()
    c = pi.pi_layer()
    ctypes.pointer(c)[0] = Lc.c
    c.w_gate_cold = None  # ReGLU needs all three
    bad = pi.Layer.__new__(pi.Layer)
    bad.__dict__.update(Lc.__dict__)
    bad.c = c
    with pytest.raises(pi.PiError) as e:
        pi.pi_ffn_stack([bad], x, 0.5, pi.PI_MASK_UNION)
    assert e.value.status == pi.PI_ERR_INVALID
    torch.cuda.synchronize()
    assert torch.equal(x, x_before)
