"""The multi-GPU path on CPU: two gloo ranks, each scanning its own batch items.

The scan shards by batch with no exchange, so the union of the ranks' outputs must
equal the single-process result exactly; the only collectives are the timing
bookkeeping (max over ranks, barrier).  The per-rank scan here is the oracle, since
this machine has no GPU; the sharding and the bookkeeping are the code under test.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from vision_mamba_selective_b200 import replicas


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist

    import oracle
    from vision_mamba_selective_b200 import workloads as wl

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    replicas.init("gloo", timeout_s=60)
    w = wl.WORKLOADS[1].scaled(batch=5, L=37, channels=16)
    x = wl.make_inputs(w)
    sl = replicas.batch_slice(w.batch, rank, world)
    y = oracle.vim_bidir(x["u"][sl], x["delta"][sl], x["z"][sl], x["B"][sl], x["C"][sl], x["A"], x["D"],
                         x["delta_bias"])
    np.save(os.path.join(out_dir, f"y{rank}.npy"), y)
    m = replicas.max_over_ranks(10.0 + rank)
    replicas.barrier()
    with open(os.path.join(out_dir, f"max{rank}.txt"), "w") as f:
        f.write(repr(m))
    dist.destroy_process_group()


def test_two_rank_batch_shards(tmp_path):
    world = 2
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    import oracle
    from vision_mamba_selective_b200 import workloads as wl

    w = wl.WORKLOADS[1].scaled(batch=5, L=37, channels=16)
    x = wl.make_inputs(w)
    full = oracle.vim_bidir(x["u"], x["delta"], x["z"], x["B"], x["C"], x["A"], x["D"], x["delta_bias"])
    parts = [np.load(tmp_path / f"y{r}.npy") for r in range(world)]
    assert [p.shape[0] for p in parts] == [3, 2]
    assert np.array_equal(np.concatenate(parts), full)
    for r in range(world):
        assert float(open(tmp_path / f"max{r}.txt").read()) == 11.0


@pytest.mark.parametrize("n,world", [(8, 1), (8, 3), (5, 2), (1, 4), (0, 2)])
def test_batch_slice_partitions(n, world):
    got = [replicas.batch_slice(n, r, world) for r in range(world)]
    idx = [i for s in got for i in range(n)[s]]
    assert idx == list(range(n))
    sizes = [len(range(n)[s]) for s in got]
    assert max(sizes) - min(sizes) <= 1


def test_rank_seeds_distinct():
    assert len({replicas.rank_seed(1002, r) for r in range(8)}) == 8
