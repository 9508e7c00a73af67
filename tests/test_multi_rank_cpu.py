"""The N > 1 path on the CPU: two `gloo` ranks (no GPU).

Checks the host logic the multi-GPU run relies on: batch shares are disjoint
and cover the batch, each rank's share computed alone equals that slice of the
full-batch result (so no data collective is needed), and the timing reduction
returns the maximum over ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from deformable_attention_sampling_b200.sharding import max_over_ranks, shard_range

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import gen
        import oracle
        w = gen.DcnWorkload("shard", N=5, H=6, W=7, C=8, G=2, dtype="f16")
        inp = gen.dcn_inputs(w, seed=3)
        start, count = shard_range(w.N, rank, world)
        part = oracle.dcn_forward_ref(inp["x"][start:start + count],
                                      inp["offset"][start:start + count],
                                      inp["mask"][start:start + count], w.kh, w.kw, w.stride,
                                      w.pad, w.dil, w.softmax_flag)
        # gather the shares (padded to the largest) on every rank
        most = shard_range(w.N, 0, world)[1]
        buf = torch.zeros((most,) + part.shape[1:], dtype=torch.float64)
        buf[:count] = torch.from_numpy(part)
        parts = [torch.zeros_like(buf) for _ in range(world)]
        dist.all_gather(parts, buf)
        counts = [shard_range(w.N, r, world)[1] for r in range(world)]
        joined = torch.cat([p[:c] for p, c in zip(parts, counts)]).numpy()
        full = oracle.dcn_forward_ref(inp["x"], inp["offset"], inp["mask"], w.kh, w.kw,
                                      w.stride, w.pad, w.dil, w.softmax_flag)
        same = bool(np.array_equal(joined, full))
        top = max_over_ranks(10.0 + rank)
        with open(os.path.join(result_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{same} {top}\n")
    finally:
        dist.destroy_process_group()


def test_shard_range_partitions_the_batch():
    for n in (0, 1, 5, 64, 127):
        for world in (1, 2, 3, 8):
            covered = []
            for r in range(world):
                s, c = shard_range(n, r, world)
                covered.extend(range(s, s + c))
            assert covered == list(range(n))
            sizes = [shard_range(n, r, world)[1] for r in range(world)]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def test_two_gloo_ranks_shard_without_data_exchange(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(WORLD, port, str(tmp_path)), nprocs=WORLD,
                       join=True, start_method="spawn")
    for r in range(WORLD):
        same, top = open(tmp_path / f"rank{r}.txt").read().split()
        assert same == "True"
        assert float(top) == 10.0 + WORLD - 1
