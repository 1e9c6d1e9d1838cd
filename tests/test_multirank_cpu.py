"""Multi-rank host logic of bench.py on CPU: two `gloo` ranks, no GPU.

With N GPUs the bench runs N replicas of the same step (weak scaling): every
rank holds the same quantized weights and its own rank-seeded activations,
and there is no data-path collective.  Checked here with world size 2:
  - the timing reduction returns the largest rank's time on every rank;
  - the whole-job value counts every rank's work;
  - the replicas' packed weights are identical and their activations differ.
"""
import hashlib
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _digest(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # timing reduction: the slowest rank's time, seen by every rank
        mine = 10.0 + 5.0 * rank
        got = bench.reduce_max(mine, world, "cpu")
        # replicas: identical packed weights, rank-seeded activations
        _, nblocks, M, projs, blocks = bench.build_host("block_m80", rank)
        w_digest = [_digest(a) for blk in blocks for p in projs for a in blk[p]]
        x_digest = [_digest(blk["x_" + p]) for blk in blocks for p in projs]
        gathered = [None] * world
        dist.all_gather_object(gathered, (w_digest, x_digest))
        flops = bench.step_flops(M, nblocks, projs)
        res = {
            "max": got,
            "weights_equal": all(g[0] == w_digest for g in gathered),
            "acts_differ": all(gathered[0][1][i] != gathered[1][1][i]
                               for i in range(len(x_digest))),
            "value": bench.job_value(world, flops, 2.0),
            "value_single": bench.job_value(1, flops, 2.0),
        }
        dist.barrier()
    finally:
        dist.destroy_process_group()
    np.save(os.path.join(out_dir, f"rank{rank}.npy"), np.array([res], dtype=object),
            allow_pickle=True)


@pytest.fixture(scope="module")
def built():
    from int8_dequant_gemm_b200 import build
    build.build()


def test_two_gloo_ranks_replicas_and_timing(tmp_path, built):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [np.load(tmp_path / f"rank{r}.npy", allow_pickle=True)[0] for r in range(world)]
    for r in res:
        assert r["max"] == 15.0                       # the slower rank's time on both
        assert r["weights_equal"] and r["acts_differ"]
        assert r["value"] == pytest.approx(2 * r["value_single"])


def test_single_rank_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.25, 1, "cpu") == 3.25
    assert bench.job_value(1, 2e12, 1000.0) == pytest.approx(2.0)
