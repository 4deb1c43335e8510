"""Failure detection on the GPU without a fault: every spin-wait in the library is
bounded, so a wait that can never end (a flag that nothing sets) gives up after
about two seconds, reports MOE_DEV_ERR_TIMEOUT in the status word, and leaves the
CUDA context usable.  The infeasible balanced plan (MOE_DEV_ERR_PLAN) is checked
in test_gpu_parity.py."""
import time

import numpy as np
import pytest
import torch

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def _buffers(s, T, k, d, E):
    n_seg, rows = moe.moe_layout(s)
    mk = lambda n, fill: torch.full((max(n, 1),), fill, dtype=torch.int32, device="cuda")
    return dict(counts=mk(E, 0), seg_expert=mk(n_seg, 0), seg_offsets=mk(n_seg + 1, 0), seg_first_rank=mk(n_seg, 0),
                dest=mk(T * k, -1), src=mk(rows, -1), xp=torch.zeros(rows, d, dtype=torch.bfloat16, device="cuda"),
                status=torch.zeros(1, dtype=torch.int32, device="cuda"))


def test_lookback_wait_that_cannot_end_times_out(cuda_ok):
    T, d, E, k = 1000, 64, 16, 2               # 2000 pairs: 8 look-back tiles
    s = moe.shape(T, d, E, k, 64)
    ids = syn.lognormal_topk_ids(E, T, k, 1.0, seed=30).cuda()
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(31)).to(torch.bfloat16).cuda()
    ws = torch.empty(moe.moe_workspace_size(s)[0], dtype=torch.uint8, device="cuda")

    b = _buffers(s, T, k, d, E)
    t0 = time.time()
    moe.moe_testing_dispatch_stalled(s, x, ids, b["counts"], b["seg_expert"], b["seg_offsets"], b["seg_first_rank"],
                                     b["dest"], b["src"], b["xp"], b["status"], ws)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert b["status"].item() & moe.DEV_ERR_TIMEOUT
    assert 1.0 < elapsed < 60.0
    assert (b["dest"].cpu().numpy() == -1).all()   # no tile could finish its look-back

    # the context is still usable: the same dispatch now gives the oracle's positions
    g = _buffers(s, T, k, d, E)
    moe.moe_dispatch(s, x, ids, 0, g["counts"], g["seg_expert"], g["seg_offsets"], g["seg_first_rank"], g["dest"],
                     g["src"], g["xp"], g["status"], ws)
    torch.cuda.synchronize()
    assert g["status"].item() == 0
    ids_np = ids.cpu().numpy()
    segs = oracle.plain_segments(oracle.histogram(ids_np, E))
    dest, _ = oracle.dispatch_positions(ids_np, segs, E)
    assert (g["dest"].cpu().numpy() == dest).all()


def test_stalled_dispatch_needs_two_tiles(cuda_ok):
    s = moe.shape(10, 64, 4, 2, 64)              # 20 pairs: a single tile, nothing would wait
    with pytest.raises(moe.MoeError):
        dummy = torch.zeros(64, dtype=torch.int32, device="cuda")
        moe.moe_testing_dispatch_stalled(s, torch.zeros(10, 64, dtype=torch.bfloat16, device="cuda"), dummy, dummy,
                                         dummy, dummy, dummy, dummy, dummy,
                                         torch.zeros(20, 64, dtype=torch.bfloat16, device="cuda"), None,
                                         torch.zeros(1 << 16, dtype=torch.uint8, device="cuda"))


def test_gemm_wait_that_cannot_end_times_out(cuda_ok):
    """The grouped GEMM's abort path: CTA 0's first pipeline stage is never filled, so its tensor-core
    issuer's wait runs out after ~2 s; the status reports the timeout, the CTA frees its tensor memory
    and returns, and a normal gate/up projection right after (which allocates all tensor memory of
    every SM it runs on) matches the oracle."""
    from gpu_cases import check_bf16_storage, make_case
    w = syn.Workload("stall", T=300, d=256, E=4, k=2, F=256, zipf_s=0.5)
    case = make_case(w, seed=40)
    ref = oracle.layer_forward(case.x, case.w_r, case.bias, case.wg, case.wu, case.wd, w.k)
    s = moe.shape(w.T, w.d, w.E, w.k, w.F)
    to_i32 = lambda a: torch.from_numpy(np.asarray(a, dtype=np.int32)).cuda()
    xp = torch.from_numpy(ref.xp.astype(np.float32)).to(torch.bfloat16).cuda()
    seg_e, seg_o = to_i32(ref.segs.expert), to_i32(ref.segs.offsets)
    wg, wu = case.wg.cuda(), case.wu.cuda()
    rows = xp.shape[0]
    hp = torch.zeros(rows, w.F, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    moe.moe_testing_gemm_stalled(s, xp, seg_e, seg_o, wg, wu, hp, st)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert st.item() & moe.DEV_ERR_TIMEOUT
    assert 1.0 < elapsed < 60.0

    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    hp2 = torch.zeros(rows, w.F, dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_gate_up(s, xp, seg_e, seg_o, wg, wu, hp2, st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    check_bf16_storage(hp2.float().cpu().numpy(), ref.hp, "Hp after the aborted GEMM")


def test_reroute_grid_barrier_that_cannot_end_times_out(cuda_ok):
    """The re-routing rounds' grid barrier: CTA 0 never arrives at the first one, so the other CTAs'
    bounded waits run out after ~2 s; the status reports the timeout and every CTA returns (the
    cooperative launch ends), and a normal re-routing dispatch right after gives the oracle's
    placement."""
    T, d, E, k, C = 1500, 64, 8, 2, 300   # 3000 pairs: three CTAs
    rng = np.random.default_rng(41)
    l = (rng.normal(size=(T, E)) - 1.2 * np.log(np.arange(1, E + 1))[None, :]).astype(np.float32)
    s = moe.shape(T, d, E, k, 64, capacity=C, route_flags=moe.ROUTE_REROUTE)
    n_seg, rows = moe.moe_layout(s)
    disp, _ = moe.moe_workspace_size(s)
    lg = torch.from_numpy(l).cuda()
    ids = torch.empty(T * k, dtype=torch.int32, device="cuda")
    wts = torch.empty(T * k, dtype=torch.float32, device="cuda")
    moe.moe_route_from_logits(s, lg, ids, wts)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(42)).to(torch.bfloat16).cuda()
    z = lambda n: torch.full((max(n, 1),), -1, dtype=torch.int32, device="cuda")
    ws = torch.empty(disp, dtype=torch.uint8, device="cuda")

    counts, se, so, sf, dest, src = z(E), z(n_seg), z(n_seg + 1), z(n_seg), z(T * k), z(rows)
    xp = torch.zeros(rows, d, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    moe.moe_testing_reroute_stalled(s, x, ids, lg, counts, se, so, sf, dest, src, xp, st, ws)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert st.item() & moe.DEV_ERR_TIMEOUT
    assert 1.0 < elapsed < 60.0

    counts, se, so, sf, dest, src = z(E), z(n_seg), z(n_seg + 1), z(n_seg), z(T * k), z(rows)
    xp = torch.zeros(rows, d, dtype=torch.bfloat16, device="cuda")
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_dispatch_reroute(s, x, ids, lg, counts, se, so, sf, dest, src, xp, st2, ws)
    torch.cuda.synchronize()
    assert st2.item() == 0
    l64 = l.astype(np.float64)
    rr = oracle.reroute_overflow(oracle.topk_ids(l64, k), l64, C)
    segs, rdest, rsrc = oracle.reroute_positions(rr)
    assert (dest.cpu().numpy() == rdest).all()
    used = int(segs.offsets[-1])
    assert (src.cpu().numpy()[:used] == rsrc).all()
    assert torch.equal(xp[:used].cpu(), x.cpu()[torch.from_numpy(rsrc // k)])
