"""The multi-rank plumbing on CPU (gloo, world size 2): blocks of the
7B-shaped model are sharded over ranks without overlap, each rank fills the
sensitivity table for its own blocks, the merged table gives every rank the
same bit allocation as one process with the whole table, and the job's time
is the maximum over ranks.  No GPU is touched (the allocation is a host
call of the library)."""
import datetime
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

N_BLOCKS = 5


def fake_scores(b, lin):
    # deterministic, distinct per linear; (tr_X, tr_G, score = tr_X tr_G)
    tx = 1.0 + 0.37 * b + 0.11 * len(lin)
    tg = 0.5 + 0.05 * ((b * 7 + len(lin) * 3) % 11)
    return (tx, tg, tx * tg)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from post_weight_quantization_syrk_b200 import dist as D
        from post_weight_quantization_syrk_b200.model import LINEARS, ModelQuantizer
        mq = ModelQuantizer(None, None, n_tokens=1, n_blocks=N_BLOCKS, device="cpu", rank=rank, world=world)
        sens = {(b, lin): fake_scores(b, lin) for b in mq.blocks for lin in LINEARS}
        alloc, full = mq.allocate(sens)
        m = D.all_max(float(10 * (rank + 1)), "cpu")
        q.put((rank, mq.blocks, sorted(alloc.items()), sorted(full.items()), m))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_and_allocation():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    blocks = [o[1] for o in out]
    assert sorted(blocks[0] + blocks[1]) == list(range(N_BLOCKS)) and not set(blocks[0]) & set(blocks[1])
    # both ranks see the full table and allocate identically
    assert out[0][2] == out[1][2] and out[0][3] == out[1][3]
    # ... and that allocation equals a single process's from the whole table
    from post_weight_quantization_syrk_b200.model import LINEARS, ModelQuantizer
    single = ModelQuantizer(None, None, n_tokens=1, n_blocks=N_BLOCKS, device="cpu")
    alloc1, full1 = single.allocate({(b, lin): fake_scores(b, lin) for b in range(N_BLOCKS) for lin in LINEARS})
    assert out[0][2] == sorted(alloc1.items())
    assert all(abs(a[1][2] - b[1][2]) == 0 for a, b in zip(out[0][3], sorted(full1.items())))
    # the job's time is the slowest rank's
    assert out[0][4] == out[1][4] == 20.0
