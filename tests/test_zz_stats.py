"""moe_routing_stats against the oracle: the routing statistics of plain, capacity and
balanced-plan layouts (the plan's figures are those of the MoonEP page's table: the busiest
group against the mean before and after planning, migrated rows, replica slots in use).
The kernel reads the oracle's tables, so only its arithmetic is under test here; the file
sorts last so that it runs after the parity tests."""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.int32))).cuda()


def _stats(s, counts, seg_expert, seg_offsets):
    out = torch.full((len(moe.STAT_NAMES),), -9, dtype=torch.int32, device="cuda")
    moe.moe_routing_stats(s, None if counts is None else _dev(counts), _dev(seg_expert), _dev(seg_offsets), out)
    torch.cuda.synchronize()
    return dict(zip(moe.STAT_NAMES, out.cpu().tolist()))


@pytest.mark.parametrize("T,E,k,sigma,C", [(1000, 16, 2, 1.0, 0), (1000, 16, 2, 1.5, 100), (333, 64, 8, 0.5, 30),
                                           (50, 8, 1, 3.0, 4)])
def test_stats_plain_and_capacity(cuda_ok, T, E, k, sigma, C):
    ids = syn.lognormal_topk_ids(E, T, k, sigma, seed=41).numpy()
    counts = oracle.histogram(ids, E)
    segs = oracle.plain_segments(counts, C)
    got = _stats(moe.shape(T, 64, E, k, 64, capacity=C), counts, segs.expert, segs.offsets)
    kept = np.minimum(counts, C) if C else counts
    assert got == dict(pairs=T * k, rows=int(kept.sum()), dropped=int(T * k - kept.sum()),
                       max_expert_load=int(counts.max()), active_experts=int((counts > 0).sum()),
                       max_segment_rows=int(kept.max()), max_group_load=int(counts.max()),
                       max_group_rows=int(kept.max()), migrated_rows=0, replicas_used=0)


@pytest.mark.parametrize("sigma", [0.0, 0.5, 1.0, 2.0, 5.0])
def test_stats_of_the_balanced_plan(cuda_ok, sigma):
    """The MoonEP experiment's shape (E = 256, R = 8, S = 2048, k = 8): after planning every group
    computes exactly S*k rows (max/mean 1.0); before, the busiest group holds max(loads)."""
    E, R, S, k, B = 256, 8, 2048, 8, 32
    T = R * S
    ids = syn.uniform_roundrobin_ids(E, T, k) if sigma == 0 else syn.lognormal_topk_ids(E, T, k, sigma, seed=42)
    counts = oracle.histogram(ids.numpy(), E)
    segs, plan = oracle.balanced_plan(counts, R, S, k, B)
    got = _stats(moe.shape(T, 64, E, k, 64, n_groups=R, replica_slots=B), counts, segs.expert, segs.offsets)
    assert got["pairs"] == got["rows"] == T * k and got["dropped"] == 0
    assert got["max_group_load"] == int(plan.loads.max())
    assert got["max_group_rows"] == S * k
    assert got["migrated_rows"] == plan.migrated_rows
    assert got["replicas_used"] == plan.replicas_used
    assert got["max_expert_load"] == int(counts.max())
    assert got["max_segment_rows"] == int(segs.length.max())
    if sigma == 0:
        assert got["migrated_rows"] == 0 and got["replicas_used"] == 0


def test_stats_without_counts_and_of_an_empty_plan(cuda_ok):
    E, R, S, k, B = 8, 4, 16, 1, 0
    s = moe.shape(R * S, 64, E, k, 64, n_groups=R, replica_slots=B)
    n_seg, _ = moe.moe_layout(s)
    # the tables an infeasible plan leaves: every segment empty
    got = _stats(s, None, np.full(n_seg, -1), np.zeros(n_seg + 1))
    assert got == dict(pairs=R * S * k, rows=0, dropped=R * S * k, max_expert_load=-1, active_experts=-1,
                       max_segment_rows=0, max_group_load=-1, max_group_rows=0, migrated_rows=0, replicas_used=0)
