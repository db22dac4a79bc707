"""The multi-GPU path on CPU: two gloo ranks exercise the rank plumbing the benchmark uses
(rank discovery, per-rank seeds, the barrier and the max-over-ranks time) and show that the
replicas are independent: each rank's result equals a single process run on its seed."""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import dist_worker  # noqa: E402
import oracle  # noqa: E402
from linear_attention_token_gdn_b200 import dist as gd  # noqa: E402
from linear_attention_token_gdn_b200 import inputs  # noqa: E402


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=dist_worker.run, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=120) for _ in procs), key=lambda d: d["rank"])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [d["rank"] for d in out] == [0, 1] and all(d["world"] == 2 and d["local"] == d["rank"] for d in out)
    assert all(d["t"] == 1.0 for d in out)            # every rank sees the slowest rank's time
    assert all(d["value"] == 64 * 2 / 1.0 for d in out)
    assert out[0]["seed"] != out[1]["seed"]
    for d in out:                                      # replica r == one process on rank r's seed
        x = inputs.make_prefill(inputs.TINY, "cpu", seed=d["seed"])
        y, _ = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"])
        assert np.isclose(float(np.abs(y).sum()), d["y_sum"], rtol=0, atol=0)
    assert out[0]["y_sum"] != out[1]["y_sum"]


def test_single_process_defaults(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert gd.env_rank() == (0, 1, 0)
    assert gd.max_over_ranks(3.5, 1) == 3.5
    assert gd.rank_seed(10, 0) == 10 and gd.rank_seed(10, 2) == 2010


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.argparse.Namespace(steps=1, warmup=3, ref_step_s=1.0)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_bench_gpus_flag_starts_the_ranks_itself():
    """`python bench.py --gpus 2` from a plain shell (no launcher environment) starts two ranks
    itself; the ranks rendezvous, reduce over each other and rank 0 reports n_gpus = 2."""
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                              "MASTER_PORT")}
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--launch-check"],
                         capture_output=True, text=True, timeout=300, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(l) for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["max_over_ranks"] == 2.0


def test_bench_rejects_a_world_size_that_differs_from_gpus():
    import subprocess
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--launch-check"],
                         capture_output=True, text=True, timeout=120, env=env)
    assert res.returncode == 2 and "WORLD_SIZE=1" in res.stderr


def test_context_parallel_gather_and_fold_on_three_gloo_ranks():
    """Context-parallel prefill's exchange and fold, on CPU: three gloo ranks each hold a
    segment of two sequences (one segment ragged), form their affine maps with the oracle,
    exchange them through the product's gather, fold the earlier ranks' maps onto S0 and run
    their segment from the folded state.  Concatenated, the segments must give the oracle's
    single pass over the whole sequences (eq. 5 makes each segment affine in its start state)."""
    segs = [64, 40, 88]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=dist_worker.run_cp, args=(r, 3, port, q, segs)) for r in range(3)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=120) for _ in procs), key=lambda d: d["rank"])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = inputs.make_prefill(inputs.TINY, "cpu", B=2, T=sum(segs), H=2, d=16, S0_std=0.05)
    y_ref, S_ref = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], x["cu_seqlens"])
    T = sum(segs)
    for d in out:
        a, b = sum(segs[:d["rank"]]), sum(segs[:d["rank"] + 1])
        n = b - a
        assert np.allclose(d["y"][:n], y_ref[a:b], rtol=1e-9, atol=1e-12)
        assert np.allclose(d["y"][n:], y_ref[T + a:T + b], rtol=1e-9, atol=1e-12)
    assert np.allclose(out[-1]["S_T"], S_ref, rtol=1e-9, atol=1e-12)
