"""Host-side checks of the benchmark harness (no GPU).

* The multi-rank path: max-over-ranks timing over a world-size-2 gloo group
  (the GPU bench uses the same function over NCCL).
* The whole-job aggregate: N ranks each doing a fixed workload (weak scaling).
* The reference arm (the fp64 oracle on the host): one JSON line from rank 0,
  nothing from other ranks.
"""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    m = bench.max_over_ranks(values[rank], dist)
    dist.barrier()
    out_q.put((rank, m))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    values = [3.25, 7.5]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, values, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 7.5, 1: 7.5}


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.25, None) == 1.25


def test_reference_arm_json_line():
    """The reference arm times the oracle on a bounded sample and reports the contract's keys."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_d64", "--steps", "2", "--warmup", "3"], capture_output=True, text=True, env=env,
                       timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["steps"] == 2 and d["warmup"] == 3


@pytest.mark.parametrize("extra, metric_tail", [(["--workload", "tiny_d64", "--dropout", "0.1"], ""),
                                                 (["--workload", "decode_b16_kv8k"], "(decode: one query per sequence)")])
def test_reference_arm_other_paths(extra, metric_tail):
    """The reference arm of the dropout step and of decode: one contract line from the oracle."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"] + extra, capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["metric"].endswith(metric_tail)
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    if "--dropout" in extra:
        assert d["config"]["dropout_p"] == 0.1 and "dropout oracle" in d["cpu_baseline"]["sample"]


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_d64", "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.parametrize("extra", [["--workload", "decode_b16_kv8k", "--dropout", "0.1"],
                                   ["--workload", "causal_n8k_d128_fp8", "--dropout", "0.1"],
                                   ["--dropout", "1.5"]])
def test_bench_rejects_dropout_where_it_does_not_apply(extra):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference"] + extra,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 2 and "--dropout" in r.stderr and r.stdout.strip() == ""


@pytest.mark.parametrize("name", ["tiny_d64", "mha_n4k_d64", "causal_n8k_d128+dropout0.1"])
def test_config_cpu_baseline(name):
    """The oracle baseline of an extra workload: a bounded sample (a fraction of a second of oracle work
    here), reported with its sample, the cores and BLAS threads, and a positive throughput."""
    sys.path.insert(0, ROOT)
    import bench
    r = bench.config_cpu_baseline(name, budget_s=0.4)
    assert r["kind"] == "oracle" and r["unit"] == "TFLOP/s" and r["value"] > 0
    assert r["cores"] >= 1 and r["cores_available"] >= 1 and "sample" in r
    if "+dropout" in name:
        assert "dropout oracle" in r["sample"]
    else:
        assert "query rows" in r["sample"]
