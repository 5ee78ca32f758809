"""The multi-GPU plumbing of bench.py (independent replicas, a barrier and the max over ranks, the
whole-job aggregate), run as two gloo ranks on the CPU.  No GPU."""
import json
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_SCRIPT = textwrap.dedent(r"""
    import contextlib, io, json, os, sys, time
    sys.path.insert(0, os.environ["REPO_ROOT"])
    import bench
    rank, world, local = bench.dist_setup(2, backend="gloo")
    # a rank that is slower than the other: the job is paced by the slowest rank
    ms = 1.0 + 2.0 * rank
    if rank == 1:
        time.sleep(0.2)
    bench.barrier_sync(world, cuda=False)
    ms_max = bench.max_over_ranks(ms, world, device="cpu")
    rate = bench.whole_job_rate(256, ms_max, world)
    # the reference arm: only rank 0 runs the oracle; the other ranks return without work
    ref_out = None
    if rank != 0:
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            t0 = time.perf_counter()
            bench.run_reference(None)  # a rank other than 0 returns before it reads its arguments
            ref_s = time.perf_counter() - t0
        ref_out = {"printed": buf.getvalue(), "seconds": ref_s}
    import torch.distributed as dist
    dist.destroy_process_group()
    print(json.dumps({"rank": rank, "world": world, "ms_max": ms_max, "rate": rate, "ref": ref_out}))
""")


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_barrier_max_and_aggregate(tmp_path):
    port = free_port()
    script = tmp_path / "rank.py"
    script.write_text(RANK_SCRIPT)
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), REPO_ROOT=ROOT, CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=240)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["world"] == 2
        assert o["ms_max"] == pytest.approx(3.0)           # max over the ranks' 1.0 and 3.0 ms
        assert o["rate"] == pytest.approx(256 * 2 * 1e3 / 3.0)  # both ranks' units over the slowest time
    ref = outs[1]["ref"]
    assert ref["printed"] == "" and ref["seconds"] < 1.0    # rank 1 of the reference arm does no work


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_setup(1) == (0, 1, 0)
    assert bench.max_over_ranks(2.5, 1) == 2.5
    assert bench.whole_job_rate(1, 0.5, 1) == pytest.approx(2000.0)
