"""World-size-2 gloo run on CPU of the multi-rank host path: each rank takes its
share of a tensor's groups (shard_desc), encodes it with the oracle, and the
gathered blocks equal the single-process encoding; the whole-job rate uses the
slowest rank's time (max over ranks, as bench.py reports)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import workloads as W
from entropy_coded_kv_b200._lib import Desc
from entropy_coded_kv_b200.shard import shard_desc, shard_range, whole_job_rate


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, blob, xb, rows, gpr, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    full = Desc(rows, gpr, gpr, gpr, 0, 0)
    d = shard_desc(full, rank, world)
    mine = xb.reshape(rows * gpr, 128)[d.src_offset: d.src_offset + d.rows * d.groups_per_row]
    blocks, _ = oracle.encode(blob, mine)
    t = torch.from_numpy(blocks.copy())
    sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(sizes, torch.tensor([t.shape[0]]))
    buf = [torch.zeros((int(s.item()), 64), dtype=torch.uint8) for s in sizes]
    dist.all_gather(buf, t)
    ms = torch.tensor([10.0 + rank], dtype=torch.float64)
    dist.all_reduce(ms, op=dist.ReduceOp.MAX)
    if rank == 0:
        out_q.put((torch.cat(buf).numpy(), float(ms.item())))
    dist.barrier()
    dist.destroy_process_group()


def test_shard_ranges_partition_exactly():
    for n in (0, 1, 7, 64, 1000):
        for world in (1, 2, 3, 8):
            got = [shard_range(n, r, world) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            assert max(b - a for a, b in got) - min(b - a for a, b in got) <= 1
    d = Desc(1, 10, 10, 10, 5, 7)
    parts = [shard_desc(d, r, 3) for r in range(3)]
    assert sum(p.groups_per_row for p in parts) == 10
    assert [p.src_offset for p in parts] == [5, 8, 11]


def test_two_gloo_ranks_reassemble_the_single_process_encoding():
    rows, gpr = 12, 3
    blob = W.random_tables(3, S_t=0.02 * 4 / 448)
    xb = np.ascontiguousarray(W.bf16_bits(W.c1_matrix()).reshape(-1)[: rows * gpr * 128])
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, blob, xb, rows, gpr, q)) for r in range(2)]
    for p in procs:
        p.start()
    got, max_ms = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want, _ = oracle.encode(blob, xb)
    np.testing.assert_array_equal(got, want)
    assert max_ms == 11.0
    assert whole_job_rate(100.0, 2, max_ms) == pytest.approx(200.0 / 0.011)
