"""Host-side logic of bench.py without a GPU: max-over-ranks timing with two
gloo ranks (the multi-GPU path is independent replicas plus this one
reduction), the clock-sample parser and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, lr = bench.dist_init("gloo")
    assert (r, w, lr) == (rank, world, rank)
    bench.barrier(w)
    got = bench.max_over_ranks(1.5 + r, w, device="cpu")
    out.put((r, got))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 2.5, 1: 2.5}


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_clock_parser(tmp_path):
    c = bench.Clocks(0)
    c.path = str(tmp_path / "c.csv")
    lines = [
        "2026/12/02 10:00:00.000, 0, 1800, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/02 10:00:00.100, 0, 1900, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/02 10:00:00.200, 0, 1700, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/02 10:00:00.300, 0, 1750, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
    ]
    open(c.path, "w").write("\n".join(lines) + "\n")

    class P:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0
    c.proc = P()
    import datetime
    t = datetime.datetime(2026, 12, 2, 10, 0, 0).timestamp()
    c.t_marks = {"warm_start": t, "timed_start": t + 0.1, "timed_end": t + 0.3}
    r = c.stop()
    assert r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"]
    assert r["sm_mhz"] == 1750


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, env=env)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny"], capture_output=True, text=True, timeout=120,
                         env=env)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_every_python_module_compiles():
    """Modules that only GPU runs import (workload, bench's GPU arm) still
    have to parse on a machine without a GPU."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    files = []
    for d in ("", "block_diffusion_speculative_softmax_b200", "oracle", "tests",
              os.path.join("tests", "golden")):
        base = os.path.join(root, d)
        files += [os.path.join(base, f) for f in os.listdir(base) if f.endswith(".py")]
    assert len(files) > 10
    for f in files:
        with open(f) as fh:
            compile(fh.read(), f, "exec")


def test_traffic_digest_ignores_comments_but_not_code():
    base = "int f(int a) {\n  return a + 1;  // one\n}\n/* block */\n"
    assert bench.code_digest(base) == bench.code_digest(base.replace("// one", "// two"))
    assert bench.code_digest(base) == bench.code_digest(base.replace("/* block */", ""))
    assert bench.code_digest(base) != bench.code_digest(base.replace("a + 1", "a + 2"))
    # every recorded DRAM traffic figure belongs to the code in this tree
    for ent in bench.TRAFFIC.values():
        assert bench.source_digest(ent["file"]).startswith(ent["sha256"])
