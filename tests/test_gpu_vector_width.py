"""Row copies and gathers move 32-byte vectors when their buffers are 32-byte aligned and 16-byte
vectors otherwise: each copying kernel (count, look-back and scatter dispatch, re-routing's row
copies, combine, expert-choice gather and combine, replica-weight prefetch, expert-parallel
dispatch) is built for both widths and launched by the alignment.
The other GPU tests allocate through torch (256-byte aligned) and so run the 32-byte kernels; here
the same calls run on buffers that start 16 bytes past a 32-byte boundary, against the oracle
(placement bit for bit, the combine to fp32 accumulation order)."""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

from gpu_cases import check_close, i32, to_np

pytestmark = pytest.mark.gpu


def buf(shape, dtype, misalign: bool):
    """A zeroed device tensor whose first element sits 16 bytes past a 32-byte boundary
    (misalign) or on one."""
    el = torch.tensor([], dtype=dtype).element_size()
    n = int(np.prod(shape))
    base = torch.zeros(n + 64 // el, dtype=dtype, device="cuda")
    want = 16 if misalign else 0
    skip = ((want - base.data_ptr() % 32) % 32) // el
    t = base[skip:skip + n].view(*shape)
    assert t.data_ptr() % 32 == want
    return t


DISPATCH = [
    # (name, T, d, E, k, capacity, R, B): the count kernel, with a capacity, the look-back kernel
    # (T*k > 65536), the grouped (expert-parallel) dispatch of a plan of at most 16 groups, the
    # count kernel with a plan of more than 16 groups, and the multi-launch plan path (more than
    # 2^20 pairs, more than 16 groups: rank + scatter kernels)
    ("count", 300, 192, 6, 2, 0, 0, 0),
    ("capacity", 500, 128, 16, 2, 40, 0, 0),
    ("lookback", 9000, 64, 64, 8, 0, 0, 0),
    ("plan-8-groups", 4096, 128, 64, 4, 0, 8, 8),
    ("plan-32-groups", 2048, 64, 64, 4, 0, 32, 8),
    ("plan-multi-launch", 140032, 64, 32, 8, 0, 32, 4),
]


@pytest.mark.parametrize("misalign", [True, False], ids=["16-byte", "32-byte"])
@pytest.mark.parametrize("name,T,d,E,k,C,R,B", DISPATCH, ids=[c[0] for c in DISPATCH])
def test_dispatch_vector_widths(cuda_ok, misalign, name, T, d, E, k, C, R, B):
    ids = syn.lognormal_topk_ids(E, T, k, 1.0, seed=21).cuda()
    s = moe.shape(T, d, E, k, 64, capacity=C, n_groups=R, replica_slots=B)
    n_seg, rows = moe.moe_layout(s)
    disp, _ = moe.moe_workspace_size(s)
    x = buf((T, d), torch.bfloat16, misalign)
    x.copy_(torch.randn(T, d, generator=torch.Generator().manual_seed(22)).to(torch.bfloat16))
    xp = buf((rows, d), torch.bfloat16, misalign)
    counts, se, so, sf, dest, src, st = i32(E), i32(n_seg), i32(n_seg + 1), i32(n_seg), i32(T * k), i32(rows), i32(1)
    moe.moe_dispatch(s, x, ids, 0, counts, se, so, sf, dest, src, xp, st,
                     torch.empty(disp, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    ids_np = ids.view(T, k).cpu().numpy()
    rc = oracle.histogram(ids_np, E)
    if R:
        segs, _ = oracle.balanced_plan(rc, R, T // R, k, B)
    else:
        segs = oracle.plain_segments(rc, C)
    rdest, rsrc = oracle.dispatch_positions(ids_np, segs, E)
    assert st.item() == 0
    assert (counts.cpu().numpy() == rc).all()
    assert (so.cpu().numpy() == segs.offsets).all()
    assert (dest.cpu().numpy() == rdest).all()
    used = int(segs.offsets[-1])
    assert (src.cpu().numpy()[:used] == rsrc[:used]).all()
    assert torch.equal(xp[:used].cpu(), x.cpu()[torch.from_numpy(rsrc[:used] // k)])


@pytest.mark.parametrize("misalign", [True, False], ids=["16-byte", "32-byte"])
def test_reroute_row_copies_vector_widths(cuda_ok, misalign):
    T, d, E, k, C = 700, 128, 9, 2, 60
    rng = np.random.default_rng(23)
    l = (rng.normal(size=(T, E)) - 1.2 * np.log(np.arange(1, E + 1))[None, :]).astype(np.float32)
    s = moe.shape(T, d, E, k, 64, capacity=C, route_flags=moe.ROUTE_REROUTE)
    n_seg, rows = moe.moe_layout(s)
    disp, _ = moe.moe_workspace_size(s)
    lg = torch.from_numpy(l).cuda()
    ids = torch.empty(T * k, dtype=torch.int32, device="cuda")
    wts = torch.empty(T * k, dtype=torch.float32, device="cuda")
    moe.moe_route_from_logits(s, lg, ids, wts)
    x = buf((T, d), torch.bfloat16, misalign)
    x.copy_(torch.randn(T, d, generator=torch.Generator().manual_seed(24)).to(torch.bfloat16))
    xp = buf((rows, d), torch.bfloat16, misalign)
    counts, se, so, sf, dest, src = i32(E), i32(n_seg), i32(n_seg + 1), i32(n_seg), i32(T * k), i32(rows)
    moe.moe_dispatch_reroute(s, x, ids, lg, counts, se, so, sf, dest, src, xp, None,
                             torch.empty(disp, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    l64 = l.astype(np.float64)
    rid = oracle.topk_ids(l64, k)
    rr = oracle.reroute_overflow(rid, l64, C)
    segs, rdest, rsrc = oracle.reroute_positions(rr)
    assert (dest.cpu().numpy() == rdest).all()
    used = int(segs.offsets[-1])
    assert (src.cpu().numpy()[:used] == rsrc).all()
    assert torch.equal(xp[:used].cpu(), x.cpu()[torch.from_numpy(rsrc // k)])


@pytest.mark.parametrize("misalign", [True, False], ids=["16-byte", "32-byte"])
@pytest.mark.parametrize("k", [2, 4, 8])
@pytest.mark.parametrize("out_dtype", ["f32", "bf16", "f32+base"])
def test_combine_vector_widths(cuda_ok, misalign, k, out_dtype):
    T, d, E = 300, 192, 8
    ids = syn.lognormal_topk_ids(E, T, k, 1.0, seed=25).numpy()
    counts = oracle.histogram(ids, E)
    segs = oracle.plain_segments(counts, 3 * T * k // (2 * E))  # drops some pairs
    dest, _ = oracle.dispatch_positions(ids, segs, E)
    rows = int(segs.offsets[-1])
    g = torch.Generator().manual_seed(26)
    yp_h, wts = torch.randn(rows, d, generator=g), torch.rand(T, k, generator=g)
    base_h = torch.randn(T, d, generator=g) if out_dtype == "f32+base" else None
    ref = oracle.combine(oracle.f64(yp_h), dest, oracle.f64(wts), T, k)
    if base_h is not None:
        ref = ref + oracle.f64(base_h)
    s = moe.shape(T, d, E, k, 64, capacity=3 * T * k // (2 * E))
    yp = buf((rows, d), torch.float32, misalign)
    yp.copy_(yp_h)
    bf16 = out_dtype == "bf16"
    if bf16:
        s.out_dtype = moe.DTYPE_BF16
    out = buf((T, d), torch.bfloat16 if bf16 else torch.float32, misalign)
    dest_d = torch.from_numpy(dest.astype(np.int32)).cuda()
    if base_h is not None:
        base = buf((T, d), torch.float32, misalign)
        base.copy_(base_h)
        moe.moe_combine_add(s, yp, dest_d, wts.cuda(), base, out)
    else:
        moe.moe_combine(s, yp, dest_d, wts.cuda(), out)
    torch.cuda.synchronize()
    if bf16:
        # one rounding of the fp32 sum to bf16
        got = to_np(out)
        assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * float(np.sqrt(np.mean(ref ** 2)))).all()
    else:
        check_close(to_np(out), ref, "out", max_abs_of_rms=1e-5, mean_rel=1e-6)


@pytest.mark.parametrize("misalign", [True, False], ids=["16-byte", "32-byte"])
def test_replica_prefetch_vector_widths(cuda_ok, misalign):
    """Rank 0 of 2 (E = 4, two experts per rank, B = 3 replica slots): slot 0 takes expert 3 (home
    rank 1), slot 1 is unused, slot 2 takes expert 2 (home rank 1) but has no rows (unused).
    Only slot 0 is written, with expert 3's matrices."""
    R, E, B, F, d = 2, 4, 3, 128, 64
    s = moe.shape(R * 64, d, E, 2, F, n_groups=R, replica_slots=B)
    n_loc = E // R + B
    g = torch.Generator().manual_seed(27)
    ws = {m: [buf((n_loc, F, d) if m != "down" else (n_loc, d, F), torch.bfloat16, misalign) for _ in range(R)]
          for m in ("gate", "up", "down")}
    for m in ws:
        for r in range(R):
            ws[m][r].copy_(torch.randn(ws[m][r].shape, generator=g).to(torch.bfloat16))
    before = {m: [t.clone() for t in ws[m]] for m in ws}
    seg_expert = torch.tensor([0, 1, 3, -1, 2], dtype=torch.int32, device="cuda")
    seg_offsets = torch.tensor([0, 5, 9, 12, 12, 12], dtype=torch.int32, device="cuda")
    moe.moe_ep_prefetch_weights(s, 0, seg_expert, seg_offsets, ws["gate"], ws["up"], ws["down"])
    torch.cuda.synchronize()
    for m in ws:
        assert torch.equal(ws[m][0][2], before[m][1][1]), m          # expert 3 = rank 1, local slot 1
        assert torch.equal(ws[m][0][:2], before[m][0][:2]), m         # home slots untouched
        assert torch.equal(ws[m][0][3:], before[m][0][3:]), m         # unused slots untouched
        assert torch.equal(ws[m][1], before[m][1]), m                 # the home rank is only read


@pytest.mark.parametrize("misalign", [True, False], ids=["16-byte", "32-byte"])
@pytest.mark.parametrize("out_dtype", ["f32", "bf16", "f32+base"])
def test_expert_choice_gather_and_combine_vector_widths(cuda_ok, misalign, out_dtype):
    """Expert choice on given scores: the selection's row gather (X -> Xp) and the combine over
    each token's rows (in column parts), on shifted or aligned buffers."""
    T, E, C, d = 900, 6, 200, 320
    rng = np.random.default_rng(28)
    S = rng.random((T, E)).astype(np.float32)
    s = moe.shape(T, d, E, 1, 64, capacity=C, route_flags=moe.ROUTE_EXPERT_CHOICE)
    n_seg, rows = moe.moe_layout(s)
    x = buf((T, d), torch.bfloat16, misalign)
    x.copy_(torch.randn(T, d, generator=torch.Generator().manual_seed(29)).to(torch.bfloat16))
    xp = buf((rows, d), torch.bfloat16, misalign)
    se, so, src, emap = i32(E), i32(E + 1), i32(rows), i32(T * E)
    row_w = torch.zeros(rows, dtype=torch.float32, device="cuda")
    moe.moe_expert_choose(s, torch.from_numpy(np.ascontiguousarray(S.T)).cuda(), x, se, so, src, row_w, emap, xp)
    torch.cuda.synchronize()
    ec = oracle.select_tokens(S, C)
    assert (src.cpu().numpy() == ec.src).all()
    assert (emap.view(T, E).cpu().numpy() == oracle.expert_choice_map(ec, T)).all()
    assert torch.equal(xp.cpu(), x.cpu()[torch.from_numpy(ec.src)])

    yp_h = torch.randn(rows, d, generator=torch.Generator().manual_seed(30))
    base_h = torch.randn(T, d, generator=torch.Generator().manual_seed(31)) if out_dtype == "f32+base" else None
    ref = oracle.combine_expert_choice(oracle.f64(yp_h), ec.src, ec.row_w.astype(np.float32), T)
    if base_h is not None:
        ref = ref + oracle.f64(base_h)
    yp = buf((rows, d), torch.float32, misalign)
    yp.copy_(yp_h)
    bf16 = out_dtype == "bf16"
    if bf16:
        s.out_dtype = moe.DTYPE_BF16
    out = buf((T, d), torch.bfloat16 if bf16 else torch.float32, misalign)
    base = None
    if base_h is not None:
        base = buf((T, d), torch.float32, misalign)
        base.copy_(base_h)
    moe.moe_combine_expert_choice(s, yp, emap, row_w, base, out)
    torch.cuda.synchronize()
    got = to_np(out)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    if bf16:
        assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * rms).all()
    else:
        check_close(got, ref, "out", max_abs_of_rms=1e-5, mean_rel=1e-6)
