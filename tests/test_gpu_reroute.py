"""Overflow re-routing on the GPU against the oracle ("Sparsely-Gated MoE 구현 관점에서
살펴보기", section "로드 밸런싱 손실(load-balancing loss)과 용량(capacity)은 별개": a pair over
its expert's capacity may go to another candidate instead of being dropped).

Placement (final expert, row, segment table, dest, src, the copied rows) is compared bit for
bit.  The candidate order comes from the fp32 logits, so the layer tests use inputs whose whole
logit order is at least 1e-3 apart for every token; the dispatch-only tests give both sides the
same synthetic fp32 logits (including many equal values and the full skewed size).
"""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

from gpu_cases import capacity_rows, check_bf16_storage, check_layer_output, check_yp_elementwise, make_case, \
    run_layer, to_np

pytestmark = pytest.mark.gpu

W = syn.Workload
SMALL = [
    W("rr-small", T=300, d=128, E=8, k=2, F=192, zipf_s=1.2, capacity_factor=0.9, reroute=True),
    W("rr-k1", T=500, d=192, E=6, k=1, F=128, zipf_s=2.0, capacity_factor=1.0, reroute=True),
    W("rr-tight", T=200, d=128, E=12, k=3, F=64, zipf_s=1.5, capacity_factor=0.5, reroute=True),   # drops remain
    W("rr-roomy", T=256, d=64, E=8, k=2, F=64, zipf_s=0.3, capacity_factor=8.0, reroute=True),     # no overflow
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_reroute_layer_matches_oracle(cuda_ok, w):
    case = make_case(w, seed=6)
    C = capacity_rows(w)
    logits, ids, wts, rr, segs, dest, src, xp, hp, yp, out = oracle.layer_forward_reroute(
        case.x, case.w_r, case.bias, case.wg, case.wu, case.wd, w.k, C)
    got = run_layer(case)
    assert got["status"] == 0
    assert (got["ids"].numpy() == ids).all()
    assert (got["counts"].numpy() == oracle.histogram(ids, w.E)).all()
    assert (got["seg_offsets"].numpy() == segs.offsets).all()
    assert (got["dest"].numpy() == dest).all()
    used = int(segs.offsets[-1])
    assert (got["src"].numpy()[:used] == src).all()
    assert (to_np(got["xp"][:used]) == xp).all()

    class R:  # the fields check_yp_elementwise reads
        pass
    r = R(); r.segs, r.hp, r.yp = segs, hp, yp
    check_bf16_storage(to_np(got["hp"][:used]), hp, "Hp")
    check_yp_elementwise(to_np(got["yp"][:used]), r, case)
    check_layer_output(to_np(got["out"]), out, dest, w.T, w.k)
    if w.name == "rr-roomy":
        assert (rr.round <= 0).all()
    else:
        assert (rr.round > 0).any(), "the case should move some pairs"


def _dispatch(T, d, E, k, C, logits32, seed):
    """ids from the GPU's top-k of the given logits, then the re-routing dispatch."""
    s = moe.shape(T, d, E, k, 64, capacity=C, route_flags=moe.ROUTE_REROUTE)
    n_seg, rows = moe.moe_layout(s)
    disp, _ = moe.moe_workspace_size(s)
    lg = torch.from_numpy(logits32).cuda()
    ids = torch.empty(T * k, dtype=torch.int32, device="cuda")
    wts = torch.empty(T * k, dtype=torch.float32, device="cuda")
    moe.moe_route_from_logits(s, lg, ids, wts)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    z = lambda n: torch.full((max(n, 1),), -7, dtype=torch.int32, device="cuda")
    counts, se, so, sf, dest, src = z(E), z(n_seg), z(n_seg + 1), z(n_seg), z(T * k), z(rows)
    xp = torch.zeros(rows, d, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(disp, dtype=torch.uint8, device="cuda")
    moe.moe_dispatch_reroute(s, x.cuda(), ids, lg, counts, se, so, sf, dest, src, xp, None, ws)
    torch.cuda.synchronize()
    return x, ids.view(T, k).cpu().numpy(), counts.cpu().numpy(), so.cpu().numpy(), dest.cpu().numpy(), \
        src.cpu().numpy(), xp


@pytest.mark.parametrize("T,E,k,C,grid", [(700, 9, 2, 60, True), (3000, 16, 4, 500, False), (400, 5, 3, 150, True)])
def test_reroute_dispatch_with_given_logits(cuda_ok, T, E, k, C, grid):
    """Logits on a coarse grid (many equal values: candidates tie and the lower id must win) or
    continuous with a Zipf-like skew; both sides take the same fp32 logits."""
    rng = np.random.default_rng(T + E)
    bias = -1.2 * np.log(np.arange(1, E + 1))
    if grid:
        l = (rng.integers(0, 5, size=(T, E)) / 4.0 + bias[None, :].round(0)).astype(np.float32)
    else:
        l = (rng.normal(size=(T, E)) + bias[None, :]).astype(np.float32)
    x, ids, counts, so, dest, src, xp = _dispatch(T, 64, E, k, C, l, seed=1)
    l64 = l.astype(np.float64)
    rid = oracle.topk_ids(l64, k)
    assert (ids == rid).all()
    rr = oracle.reroute_overflow(rid, l64, C)
    segs, rdest, rsrc = oracle.reroute_positions(rr)
    assert (counts == oracle.histogram(rid, E)).all()
    assert (so == segs.offsets).all()
    assert (dest == rdest).all()
    used = int(segs.offsets[-1])
    assert (src[:used] == rsrc).all()
    assert torch.equal(xp[:used].cpu(), x[torch.from_numpy(rsrc // k)])
    assert (rr.round > 0).any()


def test_reroute_dispatch_full_skewed_size(cuda_ok):
    """The skewed-reroute bench shape (T=8192, E=64, k=2, C=320) with synthetic fp32 logits of
    its router's scale and Zipf(1.2) bias: the whole placement bit for bit."""
    w = syn.SKEWED_REROUTE
    C = capacity_rows(w)
    rng = np.random.default_rng(11)
    l = (rng.normal(scale=1.28, size=(w.T, w.E)) - w.zipf_s * np.log(np.arange(1, w.E + 1))[None, :]).astype(np.float32)
    x, ids, counts, so, dest, src, xp = _dispatch(w.T, 256, w.E, w.k, C, l, seed=2)
    l64 = l.astype(np.float64)
    rid = oracle.topk_ids(l64, w.k)
    assert (ids == rid).all()
    rr = oracle.reroute_overflow(rid, l64, C)
    segs, rdest, rsrc = oracle.reroute_positions(rr)
    assert (so == segs.offsets).all()
    assert (dest == rdest).all()
    used = int(segs.offsets[-1])
    assert (src[:used] == rsrc).all()
    assert torch.equal(xp[:used].cpu(), x[torch.from_numpy(rsrc // w.k)])


@pytest.mark.parametrize("T,E,k", [(40000, 32, 2), (65536, 16, 8)], ids=["80k-pairs", "2^19-pairs"])
def test_reroute_dispatch_beyond_64k_pairs(cuda_ok, T, E, k):
    """More pairs than one 1024-pair slice per SM: each CTA of the grid keeps several thousand pairs
    in shared memory (the largest case is the 2^19-pair limit).  Zipf(1.2)-skewed fp32 logits, a
    capacity of the average load: the whole placement bit for bit."""
    C = T * k // E
    rng = np.random.default_rng(T + k)
    l = (rng.normal(scale=1.28, size=(T, E)) - 1.2 * np.log(np.arange(1, E + 1))[None, :]).astype(np.float32)
    x, ids, counts, so, dest, src, xp = _dispatch(T, 64, E, k, C, l, seed=3)
    l64 = l.astype(np.float64)
    rid = oracle.topk_ids(l64, k)
    assert (ids == rid).all()
    rr = oracle.reroute_overflow(rid, l64, C)
    segs, rdest, rsrc = oracle.reroute_positions(rr)
    assert (rr.round > 0).any()
    assert (so == segs.offsets).all()
    assert (dest == rdest).all()
    used = int(segs.offsets[-1])
    assert (src[:used] == rsrc).all()
    assert torch.equal(xp[:used].cpu(), x[torch.from_numpy(rsrc // k)])


def test_dispatch_rejects_the_reroute_flag(cuda_ok):
    s = moe.shape(64, 128, 8, 2, 128, capacity=16, route_flags=moe.ROUTE_REROUTE)
    dummy = torch.zeros(1 << 16, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.moe_dispatch(s, dummy, dummy, 0, dummy, dummy, dummy, dummy, dummy, dummy, dummy, None, dummy)
