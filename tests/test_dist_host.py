"""Host side of the multi-process benchmark path on CPU: two ``gloo`` ranks
(world size 2) exercise the environment parsing, the barrier, the
max-over-ranks timing and the whole-job aggregation that ``bench.py`` uses
under torchrun, plus the reference arm's rank gating. No GPU is touched."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    try:
        w, r, local = bench.dist_env()
        bench.init_dist(w, local, backend="gloo")
        bench.barrier(w)
        step_s = 1e-3 * (1 + rank)            # rank 1 is the slow one
        mx = bench.max_over_ranks(step_s, w)
        value = bench.whole_job_gbs(1e6, w, mx)
        ref = bench.run_reference(
            type("A", (), {"workload": "tiny", "warmup": 3, "steps": 1})(),
            w, r)
        bench.barrier(w)
        import torch.distributed as dist
        dist.destroy_process_group()
        q.put((rank, (w, r, local), mx, value, ref is None))
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, "error", repr(e), None, None))


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, env, mx, value, ref_none = q.get(timeout=120)
        assert env != "error", mx
        got[rank] = (env, mx, value, ref_none)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (env, mx, value, ref_none) in got.items():
        assert env == (world, rank, rank)
        assert mx == pytest.approx(2e-3)          # max over ranks
        assert value == pytest.approx(2 * 1e6 / 2e-3 / 1e9)
        assert ref_none == (rank != 0)            # only rank 0 reports


def test_single_process_defaults(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (1, 0, 0)
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_gbs(2e9, 1, 1.0) == pytest.approx(2.0)


def test_reference_arm_prints_the_contract_line():
    """``bench.py --impl reference`` (the oracle timed on the host cores on a
    bounded sample of the workload) prints one JSON line with the keys the
    benchmark contract names, on a machine without a GPU."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup",
                "ms_per_step", "higher_is_better", "scaling", "vs_baseline",
                "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1
    assert d["value"] > 0 and d["config"]["workload"] == "long"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"],
                        "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
