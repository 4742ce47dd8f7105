"""The data-parallel path with two ranks, on the CPU (gloo): each rank owns
its own batch shard (weak scaling) and the only exchange is the sum of the
weight gradients over the ranks (MicroQonv paper, section II-C3, Eq. 3: G_W
sums over the batch, so the gradient of the global batch is the sum of the
shards' gradients).  Checked against the oracle: the all-reduced G_W of two
shards equals the oracle's G_W of the concatenated batch, the step time is
the maximum over the ranks, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# one small layer, 3x3 stride 2 pad 1; each rank a shard of N_SHARD images
N_SHARD, C, H, W, K, R, S, ST, PAD = 2, 16, 9, 8, 24, 3, 3, 2, 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard(rank):
    import synth
    P, Q = (H + 2 * PAD - R) // ST + 1, (W + 2 * PAD - S) // ST + 1
    x = synth.random_tensor((N_SHARD, C, H, W), seed=500 + rank)
    g = synth.random_tensor((N_SHARD, K, P, Q), seed=600 + rank, scale=1e-3)
    return x, g


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist

    import bench
    import oracle as orc
    bench.init_dist(world, "gloo")
    x, g = _shard(rank)
    # exact (unquantized) partial gradient of this rank's shard, in double
    gw = torch.from_numpy(orc.conv_wgrad(g, x, R, S, ST, ST, PAD, PAD)[0])
    bench.allreduce_weight_grads([gw])
    np.save(os.path.join(out_dir, f"gw{rank}.npy"), gw.numpy())
    t = bench.max_over_ranks(1.5 + rank, torch.device("cpu"))
    np.save(os.path.join(out_dir, f"t{rank}.npy"), np.array([t]))
    dist.barrier()
    dist.destroy_process_group()


def test_weight_gradient_allreduce_over_two_ranks(orc, tmp_path):
    import torch.multiprocessing as mp
    mp.spawn(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    g0, g1 = np.load(tmp_path / "gw0.npy"), np.load(tmp_path / "gw1.npy")
    assert np.array_equal(g0, g1), "ranks disagree after the all-reduce"
    # the gradient of the global batch: both shards as one batch of 2 x N_SHARD
    (x0, gy0), (x1, gy1) = _shard(0), _shard(1)
    want, _ = orc.conv_wgrad(np.concatenate([gy0, gy1]), np.concatenate([x0, x1]), R, S, ST, ST, PAD, PAD)
    np.testing.assert_allclose(g0, want, rtol=1e-12, atol=1e-18)
    # the step time is the slowest rank's
    assert float(np.load(tmp_path / "t0.npy")[0]) == 2.5 and float(np.load(tmp_path / "t1.npy")[0]) == 2.5


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = bench.parse_args(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert bench.reference_arm(args) == 0
    assert capsys.readouterr().out == ""
