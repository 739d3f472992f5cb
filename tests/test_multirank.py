"""bench.py's N > 1 plumbing on CPU with the gloo backend, world size 2:
the timing barrier and max-over-ranks, the reference arm under
torch.distributed.run (rank 0 alone prints), and a rank that dies before a
collective (the other ends with an error instead of waiting forever)."""
import json
import os
import socket
import subprocess
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, die, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), PI_DIST_TIMEOUT_S="10")
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(types.SimpleNamespace(impl="reference"))
    try:
        v = bench.max_over_ranks(1.5 + r, w, "cpu")
        bench.barrier(w)
        if die and r == 1:
            os._exit(0)  # leaves between steps, without the next collective
        try:
            bench.barrier(w)
            q.put((r, v, "ok"))
        except Exception as e:  # the surviving rank's collective fails
            q.put((r, v, "error:" + type(e).__name__))
    finally:
        if not (die and r == 1):
            try:
                dist.destroy_process_group()
            except Exception:
                pass


def _run_ranks(die: bool):
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, die, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    out = {}
    while not q.empty():
        r, v, st = q.get()
        out[r] = (v, st)
    for p in procs:
        if p.is_alive():
            p.kill()
    return out


def test_barrier_and_max_over_ranks_two_ranks():
    out = _run_ranks(die=False)
    assert set(out) == {0, 1}
    for r in (0, 1):
        assert out[r][0] == 2.5  # max of 1.5 and 2.5 on every rank
        assert out[r][1] == "ok"


def test_surviving_rank_gets_an_error_when_a_rank_dies():
    out = _run_ranks(die=True)
    assert 0 in out and 1 not in out
    assert out[0][0] == 2.5
    assert out[0][1].startswith("error:"), out


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "1", "--cpu-sample-layers",
           "1", "--workload", "tiny_relu_512x2048_f32"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, PI_DIST_TIMEOUT_S="60"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    # the same config object (keys and values) the GPU arm prints for this run
    import bench
    from activation_sparse_predictor_b200 import synth
    w = synth.WORKLOADS["tiny_relu_512x2048_f32"]
    assert d["config"] == bench.run_config(w, 1, "per_token", w.n_layers, 2, "flushed")
    assert "extrapolated" in d["ms_per_step_basis"]
