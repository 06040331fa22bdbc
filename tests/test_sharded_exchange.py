"""The exchange of a KV head split across ranks, on CPU ranks (gloo, world
size 2): each rank takes the top-k of its own key range, the lists are
all-gathered, and the exact merge equals the top-k of all keys.  This is the
host side of the multi-GPU split (there, NCCL gathers and fathom_merge_topk
merges on the device)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n, k = 5000, 200
        scores = np.round(np.random.default_rng(0).standard_normal(n), 2)   # same on every rank
        bounds = [0, 2304, n]                                              # rank r owns [b_r, b_r+1)
        a, b = bounds[rank], bounds[rank + 1]
        li, ls = oracle.topk(scores[a:b], k)
        order = np.argsort(li)                                             # lists ascend by index
        mine_i = torch.from_numpy(li[order].astype(np.int32))
        mine_s = torch.from_numpy(ls[order])
        all_i = [torch.empty_like(mine_i) for _ in range(world)]
        all_s = [torch.empty_like(mine_s) for _ in range(world)]
        dist.all_gather(all_i, mine_i)
        dist.all_gather(all_s, mine_s)
        gi, _ = oracle.merge_topk(torch.stack(all_i).numpy(), torch.stack(all_s).numpy(),
                                  np.array(bounds[:-1]), k)
        ref, _ = oracle.topk(scores, k)
        out[rank] = bool(np.array_equal(gi, np.sort(ref)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_gather_and_merge_to_the_global_topk():
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res == {0: True, 1: True}
