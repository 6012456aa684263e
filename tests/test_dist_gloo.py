"""Data-parallel plumbing with two gloo ranks on CPU (no GPU): each rank gets
its own batch seed, the job's work is the sum over ranks, and the reported
time is the max over ranks.  Also checks that a rank that never joins makes
the others fail by timeout instead of hanging.
"""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _run_ranks(body, world=2, timeout=120, env_extra=None, ranks=None):
    port = _free_port()
    script = textwrap.dedent(f"""
        import os, sys, json
        sys.path.insert(0, {ROOT!r})
        import torch
        from mixed_precision_quantized_act_b200 import dist as d
        """) + textwrap.dedent(body)
    procs = []
    for r in (ranks if ranks is not None else range(world)):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE=str(world), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        env.update(env_extra or {})
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=timeout)
        except subprocess.TimeoutExpired:
            p.kill()
            out, err = p.communicate()
        outs.append((p.returncode, out, err))
    return outs


def test_two_rank_data_parallel_bookkeeping():
    outs = _run_ranks("""
        info = d.init("gloo", timeout_s=60)
        assert info.world == 2
        seed = d.batch_seed(7, info.rank)
        t = 1.0 + info.rank * 0.5          # a per-rank "device time"
        d.barrier(info.world)
        tmax = d.max_over_ranks(t, info.world)
        units = d.total_units(512, info.world)
        print(json.dumps({"rank": info.rank, "seed": seed, "tmax": tmax, "units": units}))
        d.shutdown(info.world)
    """)
    res = []
    for rc, out, err in outs:
        assert rc == 0, err
        import json
        res.append(json.loads(out.strip().splitlines()[-1]))
    assert {r["seed"] for r in res} == {7, 8}
    assert all(r["tmax"] == 1.5 for r in res)
    assert all(r["units"] == 1024 for r in res)


def test_missing_rank_times_out_instead_of_hanging():
    # only rank 0 of a world of 2 starts: its rendezvous must fail within the timeout
    outs = _run_ranks("""
        import datetime
        import torch.distributed as dist
        try:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=5))
            d.barrier(2)
            print("joined")
        except Exception as e:
            print("failed:", type(e).__name__)
    """, ranks=[0], timeout=90)
    rc, out, err = outs[0]
    assert "joined" not in out
