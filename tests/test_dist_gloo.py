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
import json

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


def test_shard_rows_cover_the_batch_once():
    sys.path.insert(0, ROOT)
    from mixed_precision_quantized_act_b200 import dist as d
    for m in (0, 1, 7, 37, 512):
        for world in (1, 2, 3, 8):
            cuts = [d.shard_rows(m, r, world) for r in range(world)]
            assert cuts[0][0] == 0 and cuts[-1][1] == m
            assert all(a[1] == b[0] for a, b in zip(cuts, cuts[1:]))
            sizes = [b - a for a, b in cuts]
            assert max(sizes) - min(sizes) <= 1


def test_two_ranks_token_shards_reassemble_the_single_rank_layer():
    """Each gloo rank quantizes and multiplies its own token shard with the
    oracle layer; the gathered A_q, s_a and Y equal one rank's result on the
    whole batch, bit for bit (the rows of a batch are independent)."""
    outs = _run_ranks("""
        import numpy as np
        import oracle
        from mixed_precision_quantized_act_b200 import workloads as wl
        info = d.init("gloo", timeout_s=60)
        layer = wl.Linear("dp_shard", 37, 200, 256, ((0, 200, 21),), 3)
        X, W, is8 = wl.make_x(layer, 4), wl.make_w(layer, 4), wl.make_bitmap(layer, 4)
        q = oracle.Quantized(W, is8)
        r0, r1 = d.shard_rows(layer.M, info.rank, info.world)
        A, s = oracle.quantize_act(X[r0:r1])
        Y = oracle.gemm_w4w8a8(A, s, q)
        A_all = d.gather_rows(torch.from_numpy(A), layer.M, info.world).numpy()
        s_all = d.gather_rows(torch.from_numpy(s), layer.M, info.world).numpy()
        Y_all = d.gather_rows(torch.from_numpy(Y), layer.M, info.world).numpy()
        A_1, s_1 = oracle.quantize_act(X)
        Y_1 = oracle.gemm_w4w8a8(A_1, s_1, q)
        ok = (np.array_equal(A_all, A_1) and np.array_equal(s_all.view(np.uint32), s_1.view(np.uint32))
              and np.array_equal(Y_all.view(np.uint16), Y_1.view(np.uint16)))
        print(json.dumps({"rank": info.rank, "rows": [r0, r1], "ok": bool(ok)}))
        d.shutdown(info.world)
    """, timeout=180)
    res = []
    for rc, out, err in outs:
        assert rc == 0, err
        res.append(json.loads(out.strip().splitlines()[-1]))
    assert sorted(tuple(r["rows"]) for r in res) == [(0, 19), (19, 37)]
    assert all(r["ok"] for r in res)


def test_bench_two_rank_dry_run_through_torchrun():
    """bench.py --gpus 2 as the driver launches it (torch.distributed.run, two
    ranks), with --dry-run: gloo instead of NCCL and no kernels, so the
    argument, rank and max-over-ranks plumbing is checked on CPU."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--gpus", "2", "--steps", "5", "--warmup", "3", "--dry-run"]
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=180, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["dry_run"] and line["world"] == 2 and line["n_gpus"] == 2
    assert line["seeds"] == [0, 1]
    assert line["ms_per_step_max_over_ranks"] == 1.25
    assert line["units"] == 2 * line["config"]["M"]
    assert line["config"]["parallelism"].startswith("dp2")
