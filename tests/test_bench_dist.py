"""Host-side checks of bench.py's multi-process path (world size 2, gloo on CPU).

Every rank runs its own replica of the workload; the bench times a step as the maximum over ranks
and reports the bytes of all ranks over that time.  These tests run the same helpers in two gloo
processes, and check that the reference arm does no work on ranks other than 0."""
import multiprocessing as mp
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


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    td, r, w, _ = bench.dist()
    try:
        bench.barrier(td)
        step_ms = 1.0 + 0.5 * rank                 # rank 1 is the slow one
        m = bench.max_over_ranks(td, step_ms)
        q.put((r, w, m, bench.job_throughput(w, 1e9, m)))
    finally:
        td.destroy_process_group()


def test_two_gloo_ranks_time_the_step_as_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[0] for o in out] == [0, 1] and all(o[1] == world for o in out)
    assert all(o[2] == pytest.approx(1.5) for o in out)          # max over ranks, seen by every rank
    assert all(o[3] == pytest.approx(2 * 1e9 / 1.5e-3 / 1e9) for o in out)  # both ranks' bytes / slowest time


def test_job_throughput_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_throughput(1, 4.5625 * 2 ** 26, 0.1) == pytest.approx(4.5625 * 2 ** 26 / 1e-4 / 1e9)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_profiles_are_consistent_with_the_bench():
    """Every committed ncu summary names a command that runs committed files (a `--case` the bench
    has), and the roofline kernel's recorded traffic equals its DRAM read + write rows."""
    import re
    sys.path.insert(0, ROOT)
    import bench
    pdir = os.path.join(ROOT, "profiles")
    for f in sorted(os.listdir(pdir)):
        text = open(os.path.join(pdir, f)).read()
        for case in re.findall(r"python bench\.py --case (\w+)", text):
            assert case in bench.CASES, (f, case)
        assert "_work" not in text, f
    t = bench.profile_traffic("nvfp4_quantize_8192x8192")
    text = open(os.path.join(pdir, "nvfp4_quantize_8192x8192.md")).read()
    four_six = text[text.index("## four-over-six"):text.index("## plain")]
    rd = float(re.search(r"DRAM read \(`dram__bytes_read\.sum`\) \| ([0-9.]+) MB", four_six).group(1))
    wr = float(re.search(r"DRAM write \(`dram__bytes_write\.sum`\) \| ([0-9.]+) MB", four_six).group(1))
    assert abs(t - (rd + wr) * 1e6) < 0.02e6


def test_oracle_is_thread_safe_for_the_all_cores_baseline():
    """The all-cores CPU baseline runs the oracle from several threads at once: each thread's
    result equals the same call made alone."""
    import concurrent.futures as cf
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle as O
    rng = np.random.default_rng(3)
    chunks = [rng.standard_normal((16, 256)).astype(np.float32) for _ in range(8)]
    serial = [O.nvfp4_quantize(c, four_six=True) for c in chunks]
    with cf.ThreadPoolExecutor(max_workers=8) as ex:
        par = list(ex.map(lambda c: O.nvfp4_quantize(c, four_six=True), chunks))
    for a, b in zip(serial, par):
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and a[2] == b[2] and a[3] == b[3]


def test_gpus_flag_spawns_the_ranks_itself():
    """`bench.py --gpus 2` without a launcher starts both ranks (gloo on a machine without a GPU);
    the helpers then see world size 2 and the slower rank's time."""
    import json
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_PORT")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dist-check"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["world"] == 2 and out["max_ms"] == pytest.approx(1.5)
    assert out["GB/s"] == pytest.approx(2 * 1e9 / 1.5e-3 / 1e9)


def test_world_size_must_match_gpus():
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "4", "--dist-check"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "WORLD_SIZE=2 but --gpus 4" in r.stderr
