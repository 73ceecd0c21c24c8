"""The multi-process host logic on CPU: world size 2 over gloo.

The quantizer shards into independent problems, so the only cross-rank steps are
bookkeeping: the max-over-ranks time of the timed region, the job's totals (values
and bytes, for the end-to-end rate) and the combination of the weighted-RMSE
accumulators.  The accumulator test splits one set of tensors
over two ranks (each rank runs the CPU oracle on its share) and checks that the
combined statistics equal the single-process ones.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from post_weight_quantization_rowwise_b200 import replicas, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        # job time: the slowest rank
        mx = replicas.max_over_ranks([1.0 + rank, 5.0 - rank])
        # job totals: values and bytes of all ranks (exact for counts below 2^53)
        tot = replicas.sum_over_ranks([1.0 + rank, 2.0 ** 40 + rank])
        # the tensor set split over ranks; each rank quantizes and scores its share
        tensors = [synth.Tensor2D(f"t{i}", 24 + 8 * i, 64, 100 + i) for i in range(5)]
        acc = torch.zeros(4, dtype=torch.float64)
        for t in replicas.shard(tensors, rank, world):
            x = t.weights().numpy()
            qw = t.qw().numpy()
            blocks, _ = oracle.quantize_q4_0_w(x, qw)
            part = oracle.weighted_rmse(x, blocks, qw)
            acc[:3] += torch.from_numpy(part[:3])
            acc[3] = max(float(acc[3]), float(part[3]))
        total = replicas.reduce_rmse(acc)
        n_mine = sum(t.numel for t in replicas.shard(tensors, rank, world))
        stats = replicas.job_rmse(acc, n_mine)  # what bench.py reports for several GPUs
        out[rank] = (mx, total.tolist(), tot, stats)
    finally:
        dist.destroy_process_group()


def test_shard_is_a_balanced_partition():
    units = list(range(11))
    parts = [replicas.shard(units, r, 4) for r in range(4)]
    assert sum(parts, []) == units
    assert max(map(len, parts)) - min(map(len, parts)) <= 1
    assert replicas.shard([], 0, 3) == []
    with pytest.raises(ValueError):
        replicas.shard(units, 4, 4)


def test_rank_seeds_differ():
    assert len({replicas.rank_seed_offset(r) for r in range(8)}) == 8
    a = synth.weight_matrix(4, 64, 7 + replicas.rank_seed_offset(0))
    b = synth.weight_matrix(4, 64, 7 + replicas.rank_seed_offset(1))
    assert not torch.equal(a, b)


def test_two_gloo_ranks_combine_like_one_process():
    import oracle
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    tensors = [synth.Tensor2D(f"t{i}", 24 + 8 * i, 64, 100 + i) for i in range(5)]
    ref = np.zeros(4)
    for t in tensors:
        x = t.weights().numpy()
        qw = t.qw().numpy()
        blocks, _ = oracle.quantize_q4_0_w(x, qw)
        oracle.weighted_rmse(x, blocks, qw, acc=ref)
    n_all = sum(t.numel for t in tensors)
    for rank in range(world):
        mx, total, tot, stats = out[rank]
        assert stats["values"] == n_all
        assert abs(stats["wrmse"] - np.sqrt(ref[0] / ref[1])) < 1e-12
        assert abs(stats["rmse"] - np.sqrt(ref[2] / n_all)) < 1e-12 and stats["maxerr"] == ref[3]
        assert mx == [2.0, 5.0]
        assert tot == [3.0, 2.0 ** 41 + 1]
        assert np.allclose(total[:3], ref[:3], rtol=1e-12, atol=0)
        assert total[3] == ref[3]
    assert abs(replicas.wrmse(out[0][1]) - np.sqrt(ref[0] / ref[1])) < 1e-12
