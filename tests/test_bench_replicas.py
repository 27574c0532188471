"""bench.py's multi-GPU mode runs replicas: every rank runs the same workload with no
collective on the data path. The reported time is the maximum over ranks, and `value` is
the bytes of all ranks divided by that time. Two gloo ranks on the CPU drive bench.py's own
max_over_ranks and replica_value with different per-rank times."""
import os

import pytest
import torch.multiprocessing as mp

import bench


def _rank(rank: int, world: int, port: int, out) -> None:
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [[1000.0, 300.0], [1500.0, 200.0]][rank]  # (timed steps, e2e) device µs
        total_us, e2e_us = bench.max_over_ranks(mine, world, "cpu")
        out[rank] = (total_us, e2e_us, bench.replica_value(1e6, 10, world, total_us))
    finally:
        dist.destroy_process_group()


def test_replicas_report_max_over_ranks():
    world, port = 2, 29517
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        total_us, e2e_us, value = out[r]
        assert (total_us, e2e_us) == (1500.0, 300.0)
        assert value == pytest.approx(2 * 1e6 * 10 / 1500e-6 / 1e9)


def test_single_rank_is_unchanged():
    assert bench.max_over_ranks([5.0, 7.0], 1) == [5.0, 7.0]
    assert bench.replica_value(2e9, 1, 1, 1e6) == pytest.approx(2.0)


def test_algorithmic_bytes_formula():
    # n*k/2 codes + n*k/16 scales + 2*m*k activations + 2*m*n outputs
    assert bench.algorithmic_bytes(1, 4096, 14336) == 33_067_008
    assert bench.algorithmic_bytes(1, 512, 2048) == 594_944


def test_traffic_hash_ignores_comments_only():
    """The stored DRAM-traffic figures are keyed by the kernel code with comments removed:
    comment edits keep the key, a code edit (even inside a PTX string) changes it."""
    src = ('// header\n#include "a.h"\n/* block\n comment */ int x = 1; // trailing\n'
           'asm("mov.b32 %0, %1; // not a comment");\n')
    stripped = bench._strip_comments(src)
    assert stripped == '#include "a.h"\n int x = 1;\nasm("mov.b32 %0, %1; // not a comment");'
    assert bench._strip_comments(src.replace("trailing", "other words")) == stripped
    assert bench._strip_comments(src.replace("int x = 1", "int x = 2")) != stripped
    assert bench._strip_comments(src.replace("%0, %1", "%1, %0")) != stripped
