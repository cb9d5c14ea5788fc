"""The multi-rank plumbing on CPU (gloo, world sizes 2 and 3): blocks of the
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


@pytest.mark.parametrize("world", [2, 3])
def test_rank_sharding_and_allocation(world):
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
    # every block on exactly one rank
    assert sorted(b for bl in blocks for b in bl) == list(range(N_BLOCKS))
    assert all(not set(blocks[i]) & set(blocks[j]) for i in range(world) for j in range(i))
    # every rank sees the full table and allocates identically
    assert all(o[2] == out[0][2] and o[3] == out[0][3] for o in out)
    # ... and that allocation equals a single process's from the whole table
    from post_weight_quantization_syrk_b200.model import LINEARS, ModelQuantizer
    single = ModelQuantizer(None, None, n_tokens=1, n_blocks=N_BLOCKS, device="cpu")
    alloc1, full1 = single.allocate({(b, lin): fake_scores(b, lin) for b in range(N_BLOCKS) for lin in LINEARS})
    assert out[0][2] == sorted(alloc1.items())
    assert all(abs(a[1][2] - b[1][2]) == 0 for a, b in zip(out[0][3], sorted(full1.items())))
    # the job's time is the slowest rank's
    assert all(o[4] == 10.0 * world for o in out)
