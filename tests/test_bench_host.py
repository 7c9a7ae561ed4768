"""Host-side logic of bench.py: the reference (oracle) arm's JSON line, the
rank plumbing under torch.distributed with world_size 2 (gloo, CPU), and the
workload byte accounting."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "fp8_single", "--steps", "3", "--warmup", "1"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "workload" in d["config"]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    r = bench.Ranks()
    r.init("gloo")
    r.barrier()
    m = r.max(float(10 + rank), "cpu")
    q.put((rank, m))
    r.close()


def test_ranks_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(i, 2, port, q)) for i in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 11.0, 1: 11.0}


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.parse_args(["--impl", "reference", "--workload", "fp8_single", "--steps", "1", "--warmup", "0"])
    bench.run_reference(args, bench.Ranks())
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("name,per_elem", [("grouped_moe", 3.125), ("grouped_moe_amax_given", 3.125),
                                           ("grouped_moe_row_rht", 3.125), ("grouped_moe_sr", 3.125), ("dense_nvfp4", 3.125), ("dsa_indexer", 3.03125),
                                           ("dsa_indexer_nvfp4", 2.59375),
                                           ("qmoe_bf16", 3.03125), ("qmoe_swiglu", 9.03125)])
def test_algorithmic_bytes(name, per_elem):
    wl = bench.make_workload(name, 0)
    extra = 16 * len(wl.splits) if hasattr(wl, "splits") else 0
    assert wl.alg_bytes() == int(wl.elements() * per_elem) + extra


def test_grouped_config_matches_the_headline_workload():
    wl = bench.make_workload("grouped_moe", 0)
    assert (wl.M, wl.K, len(wl.splits), sum(wl.splits)) == (16384, 7168, 32, 16384)
    assert wl.splits[0] == 0 and wl.splits[1] == 128 and all(s % 128 == 0 for s in wl.splits)
    assert wl.alg_bytes() == 367_001_600 + 512
