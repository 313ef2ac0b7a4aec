"""World-size-2 checks of bench.py's multi-rank host logic on CPU (gloo).

The layer is token-parallel: each rank runs its own shard of tokens with the
replicated weights and no collective on the forward data path.  What the ranks
share is the timing reduction (max over ranks) and the whole-job throughput;
the weight gradient of a data-parallel step adds one exchange, the sum of the
ranks' dW (bench.reduce_weight_grad).
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads as synth
        # max over ranks of per-rank timings
        got = bench.max_over_ranks([10.0 + rank, 5.0 - rank], torch.device("cpu"))
        # each rank's shard: same shape, different tokens
        w = synth.CYCLIC_WORKLOADS["c4_t64_16x16_f32"]
        x, W = synth.cyclic_inputs(w.T, w.Cin, w.Cout, w.N, w.torch_dtype, bench.rank_seed(w, rank))
        xs = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(xs, x)
        Ws = [torch.empty_like(W) for _ in range(world)]
        dist.all_gather(Ws, W)
        out[rank] = (got, all(t.shape == x.shape for t in xs), not torch.equal(xs[0], xs[1]))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_shards():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        got, same_shape, distinct = out[r]
        assert got == [11.0, 5.0]          # element-wise max over both ranks
        assert same_shape and distinct     # equal shard shapes, different tokens


def test_single_process_reduction_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]


def test_job_throughput_counts_every_rank():
    import bench
    # 4 ranks x 1000 tokens x 10 steps in 20 ms of the slowest rank
    assert bench.job_tokens_per_s(1000, 4, 10, 20.0) == pytest.approx(2.0e6)


def _wgrad_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import numpy as np
        import bench
        import oracle
        import workloads as synth
        w = synth.CYCLIC_WORKLOADS["c4_t64_16x16_f32"]
        x, _, dy = synth.cyclic_backward_inputs(w.T, w.Cin, w.Cout, w.N, torch.float64, bench.rank_seed(w, rank))
        dW = torch.from_numpy(oracle.cyclic_weight_grad(x.numpy(), dy.numpy()))
        bench.reduce_weight_grad(dW)
        xs = [torch.empty_like(x) for _ in range(world)]
        dys = [torch.empty_like(dy) for _ in range(world)]
        dist.all_gather(xs, x)
        dist.all_gather(dys, dy)
        whole = oracle.cyclic_weight_grad(torch.cat(xs).numpy(), torch.cat(dys).numpy())
        out[rank] = float(np.max(np.abs(dW.numpy() - whole)) / np.max(np.abs(whole)))
    finally:
        dist.destroy_process_group()


def test_two_rank_weight_gradient_is_the_whole_batch_gradient():
    """The sum over ranks of each shard's dW is the gradient over all ranks' tokens."""
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_wgrad_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        assert out[r] < 1e-12


_PROBE = r"""
import datetime, os, sys
import torch, torch.distributed as dist
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
t = torch.tensor([float(dist.get_rank() + 1)])
dist.all_reduce(t)
print(f"rank={dist.get_rank()} world={dist.get_world_size()} sum={t.item():g} args={sys.argv[1:]}", flush=True)
dist.destroy_process_group()
"""


def test_bench_launcher_starts_one_rank_per_gpu(tmp_path):
    """bench.py --gpus N started as one process re-launches itself as N ranks
    through launcher_command; here the same command runs a 2-rank gloo probe."""
    import subprocess
    import sys
    import bench
    probe = tmp_path / "probe.py"
    probe.write_text(_PROBE)
    cmd = bench.launcher_command(["--gpus", "2", "--steps", "3"], 2, _free_port(), script=str(probe))
    assert cmd[:3] == [sys.executable, "-m", "torch.distributed.run"]
    assert "--nproc-per-node=2" in cmd and "127.0.0.1" in cmd
    env = dict(os.environ, OMP_NUM_THREADS="1")
    env.pop("WORLD_SIZE", None)
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=240, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    import re
    # the ranks share one stdout, so their lines may interleave: match each record
    got = sorted(re.findall(r"rank=\d world=\d sum=\d args=\[[^\]]*\]", out.stdout))
    assert got == [f"rank={r} world=2 sum=3 args=['--gpus', '2', '--steps', '3']" for r in range(2)]
