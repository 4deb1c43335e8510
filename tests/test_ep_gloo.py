"""Expert parallelism, host side, on two gloo ranks (CPU): the counts exchange gives every rank
the same [R, E] table in rank order, so every rank computes the same balanced plan -- the plan
of all R*S tokens in rank order -- and the address exchange gives every rank the same table of
peer addresses in rank order.  The device kernels are checked on one GPU with virtual ranks
(tests/test_gpu_ep.py)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from mixture_experts_routing_02_b200 import ep
from mixture_experts_routing_02_b200 import synthetic as syn

R, S, E, K, B = 2, 300, 16, 4, 6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ids(rank):
    return syn.lognormal_topk_ids(E, S, K, 1.5, seed=100 + rank).numpy()


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        counts = torch.from_numpy(oracle.histogram(_ids(rank), E).astype(np.int32))
        counts_all = ep.gather_counts(counts)
        segs, _ = oracle.balanced_plan(counts_all.sum(0).numpy(), R, S, K, B)
        addresses = ep.gather_addresses((rank + 1) << 20)
        q.put((rank, counts_all.numpy(), segs.expert, segs.offsets, segs.first_rank, addresses))
    finally:
        dist.destroy_process_group()


def test_counts_exchange_and_plan_agreement_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, R, port, q)) for r in range(R)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in range(R)], key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ids_all = np.concatenate([_ids(r) for r in range(R)])
    want_counts = np.stack([oracle.histogram(_ids(r), E) for r in range(R)])
    want_segs, _ = oracle.balanced_plan(oracle.histogram(ids_all, E), R, S, K, B)
    for rank, counts_all, seg_e, seg_o, seg_f, addresses in res:
        assert (counts_all == want_counts).all(), f"rank {rank}: gathered counts"
        assert (seg_e == want_segs.expert).all() and (seg_o == want_segs.offsets).all()
        assert (seg_f == want_segs.first_rank).all()
        assert addresses == [1 << 20, 2 << 20]
    # every rank's group holds exactly S*k rows of the plan of all tokens in rank order
    pg = E // R + B
    assert (np.diff(want_segs.offsets[::pg]) == S * K).all()
