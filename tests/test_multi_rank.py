"""World-size-2 runs of the multi-GPU bookkeeping in bench.py on CPU (gloo).

The layer shards across GPUs as independent replicas (same weights, a
different batch per rank, no data-path collective); what has to be right for
N > 1 is the host side: rank/world parsing, the max-over-ranks time and the
sum-over-ranks token count that form the whole-job throughput, per-rank batch
seeds, and the reference arm running on rank 0 only.  No GPU is involved."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    from routing_dispatch_expert_softmax_b200 import workloads as wl

    r, w, local = bench.dist_env()
    dist = bench.init_dist(w, "gloo")
    try:
        # rank r "took" (r + 1) ms per step over 3 steps and did T tokens per step
        t_max = bench.max_over_ranks(dist, 3.0 * (r + 1), "cpu")
        tokens = bench.sum_over_ranks(dist, 64 * 3, "cpu")
        cfg = wl.TINY
        x = wl.make_hidden(cfg, "cpu", r)
        w13, _ = wl.make_experts(cfg, "cpu", 0)
        x_all = [torch.empty_like(x) for _ in range(w)]
        dist.all_gather(x_all, x)
        w_all = [torch.empty_like(w13) for _ in range(w)]
        dist.all_gather(w_all, w13)
        out[r] = dict(rank=r, world=w, local=local, t_max=t_max, tokens=tokens,
                      x_differ=not torch.equal(x_all[0], x_all[1]),
                      w_same=torch.equal(w_all[0], w_all[1]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _ref_worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import contextlib
    import io

    import bench
    args = bench.parse_args(["--gpus", str(world), "--steps", "1", "--warmup", "1",
                             "--workload", "tiny"])
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.run_reference(args)
    out[rank] = (rc, buf.getvalue())


def _spawn(fn, world=2):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(fn, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        return dict(out)


def test_two_rank_throughput_bookkeeping():
    res = _spawn(_worker)
    assert sorted(res) == [0, 1]
    for r, v in res.items():
        assert (v["rank"], v["world"], v["local"]) == (r, 2, r)
        assert v["t_max"] == pytest.approx(6.0)      # the slower rank's time
        assert v["tokens"] == pytest.approx(2 * 192)  # every rank's tokens
        assert v["x_differ"] and v["w_same"]          # replicas: own batch, same weights


def test_reference_arm_runs_on_rank_zero_only():
    res = _spawn(_ref_worker)
    rc0, out0 = res[0]
    rc1, out1 = res[1]
    assert rc0 == 0 and rc1 == 0
    assert '"impl": "reference"' in out0
    assert out1.strip() == ""


def test_routing_stats_against_the_oracle_imbalance_factor():
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    import oracle
    rng = np.random.default_rng(0)
    for E, R in ((8, 4), (256, 8), (128, 0), (6, 1)):
        counts = torch.from_numpy(rng.integers(0, 50, E).astype(np.int32))
        st = bench.routing_stats(counts.tolist(), R)
        c = counts.numpy()
        assert st["rows"] == int(c.sum())
        assert st["touched_experts"] == int((c > 0).sum())
        assert st["max_rows_per_expert"] == int(c.max())
        assert st["mean_rows_per_expert"] == c.sum() / E
        if R > 1:
            assert st["rows_per_rank"] == c.reshape(R, -1).sum(1).tolist()
            assert st["imbalance_factor"] == oracle.imbalance_factor(c, R)
        else:
            assert "imbalance_factor" not in st
    assert bench.routing_stats([0, 0, 0, 0], 2)["imbalance_factor"] == 0.0


@pytest.mark.parametrize("extra", [[], ["--fp8"]])
def test_reference_arm_line_on_cpu(extra):
    import json
    import subprocess
    import sys
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "0", *extra],
                         capture_output=True, text=True, env=env, timeout=600, check=True).stdout
    line = json.loads(out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert ("weights" in line["config"]) == bool(extra)
