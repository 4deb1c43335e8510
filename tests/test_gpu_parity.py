"""GPU-vs-oracle parity of every C-ABI call on small, ragged and degenerate
cases (the oracle finishes each in seconds; the cases span several tiles and
leave ragged tails).  Integer and index outputs must match bit for bit;
floating-point outputs must meet the tolerance in ``gpu_cases.check_close``.
"""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

from gpu_cases import (check_yp_elementwise, Case, check_bf16_storage, check_close, check_layer_output, dev, i32, make_case, moe_shape,
                       oracle_segments, run_layer, to_np)

pytestmark = pytest.mark.gpu

SMALL = [
    syn.TINY,
    syn.Workload("ragged", T=300, d=192, E=6, k=2, F=320, zipf_s=1.2),
    syn.Workload("many-experts", T=333, d=256, E=64, k=8, F=128),
    syn.Workload("capacity", T=500, d=128, E=16, k=2, F=192, zipf_s=1.2, capacity_factor=1.0),
    syn.Workload("capacity-1", T=40, d=64, E=4, k=2, F=64, capacity_factor=0.05),
    syn.Workload("plan", T=512, d=128, E=16, k=4, F=128, zipf_s=1.2, n_groups=4, replica_slots=8),
    syn.Workload("dense-e1k1", T=130, d=64, E=1, k=1, F=64),
    syn.Workload("k-equals-e", T=77, d=128, E=8, k=8, F=128),
    syn.Workload("one-token", T=1, d=64, E=4, k=2, F=64),
    syn.Workload("multi-tile", T=1000, d=512, E=4, k=2, F=512, zipf_s=0.5),
    syn.Workload("wide-router", T=260, d=128, E=256, k=6, F=64),
    # long segments: several 128-row tiles per expert, ragged tails
    syn.Workload("long-ragged", T=700, d=192, E=3, k=2, F=320, zipf_s=1.0),
    syn.Workload("long-plan", T=2048, d=128, E=8, k=2, F=128, zipf_s=1.2, n_groups=2, replica_slots=4),
    syn.Workload("long-capacity", T=1500, d=256, E=4, k=2, F=192, zipf_s=1.2, capacity_factor=1.0),
    syn.Workload("long-small", T=600, d=64, E=2, k=1, F=64),
    # dispatch paths by size: T*k = 65536 is the largest for the single-pass count kernel; above
    # it the look-back kernel runs (with and without a capacity)
    syn.Workload("count-largest", T=8192, d=64, E=16, k=8, F=64, zipf_s=0.7),
    syn.Workload("lookback", T=9000, d=64, E=64, k=8, F=64, zipf_s=0.5),
    syn.Workload("lookback-capacity", T=9000, d=64, E=32, k=8, F=64, zipf_s=1.2, capacity_factor=1.0),
]


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    moe.load_library()


def _oracle_layer(case: Case):
    w = case.w
    C = oracle.capacity_rows(w.capacity_factor, w.T, w.k, w.E)
    return oracle.layer_forward(case.x, case.w_r, case.bias, case.wg, case.wu, case.wd, w.k,
                                capacity=C, n_groups=w.n_groups, replica_slots=w.replica_slots)


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_layer_matches_oracle(w):
    case = make_case(w, seed=1)
    ref = _oracle_layer(case)
    got = run_layer(case)
    assert got["status"] == 0
    # routing: ids bit-exact, weights to fp32 accuracy
    assert (got["ids"].numpy() == ref.ids).all(), "top-k ids differ"
    assert np.abs(got["w"].numpy() - ref.weights).max() < 1e-4
    # dispatch: counts, segment tables, positions bit-exact
    assert (got["counts"].numpy() == ref.counts).all()
    assert (got["seg_expert"].numpy() == ref.segs.expert).all()
    assert (got["seg_offsets"].numpy() == ref.segs.offsets).all()
    assert (got["seg_first_rank"].numpy() == ref.segs.first_rank).all()
    assert (got["dest"].numpy() == ref.dest).all()
    used = int(ref.segs.offsets[-1])
    assert (got["src"].numpy()[:used] == ref.src).all()
    # permuted rows are exact copies
    assert (to_np(got["xp"][:used]) == ref.xp).all()
    # expert FFN and combine within tolerance of the fp64 oracle
    check_bf16_storage(to_np(got["hp"][:used]), ref.hp, "Hp")
    check_yp_elementwise(to_np(got["yp"][:used]), ref, case)
    check_layer_output(to_np(got["out"]), ref.out, ref.dest, w.T, w.k)


BF16_OUT = ["tiny", "ragged", "capacity", "plan", "one-token", "count-largest", "lookback-capacity"]

# Small layers whose bf16 output misses max-abs <= 2e-2 x RMS (measured on B200): the fp32 output
# meets it, and rounding to bf16 adds up to half a bf16 ulp (2^-9 |out|) at the largest outputs.
BF16_MISSES = {"plan": "max-abs 2.12e-2 x RMS", "count-largest": "max-abs 2.09e-2 x RMS",
               "lookback-capacity": "max-abs 3.10e-2 x RMS"}


@pytest.mark.parametrize("name", BF16_OUT)
def test_layer_bf16_output_is_the_rounded_fp32_output(name):
    """out_dtype = bf16: the layer output is the fp32 combine rounded once to bf16 (round to nearest
    even), bit for bit; fully dropped tokens are exactly 0."""
    w = next(x for x in SMALL if x.name == name)
    case = make_case(w, seed=1)
    f32 = run_layer(case)
    b16 = run_layer(case, out_dtype=moe.DTYPE_BF16)
    assert f32["status"] == 0 and b16["status"] == 0
    assert b16["out"].dtype == torch.bfloat16
    assert torch.equal(b16["out"], f32["out"].to(torch.bfloat16)), "bf16 output is not the rounded fp32 output"


@pytest.mark.parametrize("name", [pytest.param(n, marks=pytest.mark.xfail(
    reason="measured miss of the stated tolerance with a bf16 output: " + BF16_MISSES[n], strict=False))
    if n in BF16_MISSES else n for n in BF16_OUT])
def test_layer_bf16_output_tolerance(name):
    """The bf16 output against the fp64 oracle with the stated tolerance (listed misses reported as
    expected failures)."""
    w = next(x for x in SMALL if x.name == name)
    case = make_case(w, seed=1)
    ref = _oracle_layer(case)
    b16 = run_layer(case, out_dtype=moe.DTYPE_BF16)
    assert b16["status"] == 0
    check_layer_output(to_np(b16["out"]), ref.out, ref.dest, w.T, w.k, "bf16 out")


def test_combine_add_and_expert_choice_bf16_output():
    """moe_combine_add and moe_combine_expert_choice with a bf16 out: the fp32 results rounded once;
    a bf16 out aliasing the fp32 base is rejected."""
    w = syn.Workload("combine-bf16", T=257, d=192, E=6, k=3, F=64, zipf_s=1.0, capacity_factor=0.8)
    s32 = moe_shape(w)
    s16 = moe_shape(w)
    s16.out_dtype = moe.DTYPE_BF16
    n_seg, rows = moe.moe_layout(s32)
    g = torch.Generator(device="cuda").manual_seed(5)
    yp = torch.randn(rows, w.d, device="cuda", generator=g)
    base = torch.randn(w.T, w.d, device="cuda", generator=g)
    wts = torch.rand(w.T, w.k, device="cuda", generator=g)
    dest = torch.randint(-1, rows, (w.T * w.k,), device="cuda", dtype=torch.int32, generator=g)
    o32 = torch.empty(w.T, w.d, device="cuda")
    o16 = torch.empty(w.T, w.d, device="cuda", dtype=torch.bfloat16)
    moe.moe_combine_add(s32, yp, dest, wts, base, o32)
    moe.moe_combine_add(s16, yp, dest, wts, base, o16)
    torch.cuda.synchronize()
    assert torch.equal(o16, o32.to(torch.bfloat16))
    with pytest.raises(moe.MoeError):
        moe.moe_combine_add(s16, yp, dest, wts, base, base)

    e = syn.Workload("ec-bf16", T=300, d=128, E=8, k=2, F=64, capacity_factor=1.0, expert_choice=True)
    case = make_case(e, seed=4)
    ref32 = run_layer(case)
    got16 = run_layer(case, out_dtype=moe.DTYPE_BF16)
    assert ref32["status"] == 0 and got16["status"] == 0
    assert torch.equal(got16["out"], ref32["out"].to(torch.bfloat16))


def test_layer_softmax_all_variant():
    """The whole layer with weights from a softmax over all experts (no renormalisation)."""
    w = syn.Workload("softmax-all", T=300, d=192, E=16, k=4, F=128, zipf_s=0.8)
    case = make_case(w, seed=13)
    ref = oracle.layer_forward(case.x, case.w_r, case.bias, case.wg, case.wu, case.wd, w.k, softmax_all=True)
    got = run_layer(case, route_flags=moe.ROUTE_SOFTMAX_ALL)
    assert got["status"] == 0
    assert (got["ids"].numpy() == ref.ids).all()
    assert np.abs(got["w"].numpy() - ref.weights).max() < 1e-5
    assert (got["w"].numpy().sum(1) < 1).all()
    check_layer_output(to_np(got["out"]), ref.out, ref.dest, w.T, w.k)


@pytest.mark.parametrize("E,flags", [(5, 0), (24, 0), (32, 0), (33, 0), (40, 0), (256, 0), (8, 1), (256, 1)])
def test_route_logits_and_bias(E, flags):
    """The tensor-core router with N = E padded to a multiple of 16 (E = 5 ... 256); flags = 1 is
    the softmax over all E without renormalisation."""
    w = syn.Workload("route", T=333, d=320, E=E, k=min(5, E), F=64, zipf_s=1.2)
    case = make_case(w, seed=2)
    s = moe_shape(w)
    s.route_flags = flags
    logits = torch.empty(w.T, w.E, device="cuda")
    ids = i32(w.T * w.k).view(w.T, w.k)
    wt = torch.empty(w.T, w.k, device="cuda")
    st = i32(1)
    moe.moe_route(s, dev(case.x), dev(case.w_r), dev(case.bias), logits, ids, wt, st)
    torch.cuda.synchronize()
    l64, rid, rw = oracle.route(case.x, case.w_r, case.bias, w.k, softmax_all=bool(flags))
    check_close(to_np(logits), l64, "logits", max_abs_of_rms=1e-4, mean_rel=1e-5)
    assert (ids.cpu().numpy() == rid).all()
    assert np.abs(wt.cpu().numpy() - rw).max() < 1e-4
    assert st.item() == 0


@pytest.mark.parametrize("E,flags", [(8, 0), (60, 1), (256, 0)])
def test_route_split_reduction(E, flags):
    """moe_route_ws: the router projection's reduction split over more CTAs (partial logits in
    the workspace, summed in order by a second kernel) gives the oracle's routing, and exactly the
    routing of moe_route_from_logits on the logits it wrote."""
    w = syn.Workload("route-split", T=900, d=1024, E=E, k=min(6, E), F=64, zipf_s=1.2)
    case = make_case(w, seed=3)
    s = moe_shape(w)
    s.route_flags = flags
    n = moe.moe_route_workspace_size(s)
    assert n > 0, "this shape should split the reduction"
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    logits = torch.empty(w.T, w.E, device="cuda")
    ids = i32(w.T * w.k).view(w.T, w.k)
    wt = torch.empty(w.T, w.k, device="cuda")
    st = i32(1)
    moe.moe_route_ws(s, dev(case.x), dev(case.w_r), dev(case.bias), logits, ids, wt, st, ws)
    torch.cuda.synchronize()
    l64, rid, rw = oracle.route(case.x, case.w_r, case.bias, w.k, softmax_all=bool(flags))
    check_close(to_np(logits), l64, "logits", max_abs_of_rms=1e-4, mean_rel=1e-5)
    assert (ids.cpu().numpy() == rid).all()
    assert np.abs(wt.cpu().numpy() - rw).max() < 1e-4
    assert st.item() == 0
    ids_l = i32(w.T * w.k).view(w.T, w.k)
    wt_l = torch.empty(w.T, w.k, device="cuda")
    moe.moe_route_from_logits(s, logits, ids_l, wt_l)
    torch.cuda.synchronize()
    assert torch.equal(ids_l, ids) and torch.equal(wt_l, wt), "fused routing differs from routing its logits"
    # without a workspace the same call runs the single-pass kernel
    ids2 = i32(w.T * w.k).view(w.T, w.k)
    moe.moe_route_ws(s, dev(case.x), dev(case.w_r), dev(case.bias), None, ids2, wt, st, None)
    torch.cuda.synchronize()
    assert torch.equal(ids2, ids)


def test_route_scores_split_reduction():
    """moe_route_scores_ws (expert choice) with the split reduction against the oracle's scores."""
    w = syn.Workload("ec-split", T=700, d=768, E=16, k=2, F=64, capacity_factor=1.0, expert_choice=True)
    case = make_case(w, seed=4)
    s = moe_shape(w)
    n = moe.moe_route_workspace_size(s)
    assert n > 0
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    scores = torch.empty(w.E, w.T, device="cuda")
    st = i32(1)
    moe.moe_route_scores_ws(s, dev(case.x), dev(case.w_r), dev(case.bias), scores, st, ws)
    torch.cuda.synchronize()
    ref = oracle.expert_scores(oracle.router_logits(case.x, case.w_r, case.bias))
    got = scores.cpu().numpy().T
    assert (np.abs(got - ref) <= 1e-4 * ref + 1e-9).all()
    assert st.item() == 0


@pytest.mark.parametrize("flags", [0, 1])
def test_route_from_logits_ties_and_exact_decision(flags):
    T, E, k = 97, 37, 6
    rng = np.random.default_rng(5)
    l = rng.normal(size=(T, E)).astype(np.float32)
    l[:, 7] = l[:, 3]            # exact ties: the lower id must come first
    l[:10, :] = 1.0              # rows of all-equal logits
    l[10, :] = np.float32(-3.0)
    l[10, 20] = 2.0
    s = moe.shape(T, 64, E, k, 64, route_flags=flags)
    ids = i32(T * k).view(T, k)
    wt = torch.empty(T, k, device="cuda")
    moe.moe_route_from_logits(s, torch.from_numpy(l).cuda(), ids, wt)
    torch.cuda.synchronize()
    l64 = l.astype(np.float64)
    rid = oracle.topk_ids(l64, k)
    assert (ids.cpu().numpy() == rid).all()
    ref_w = oracle.topk_weights_softmax_all(l64, rid) if flags else oracle.topk_weights(l64, rid)
    assert np.abs(wt.cpu().numpy() - ref_w).max() < 1e-6
    assert list(ids.cpu().numpy()[0]) == list(range(k))


def test_worked_example_on_the_gpu():
    """The worked top-2 example (E4 = 2.0, E6 = 1.6 -> ids 3, 5, weights 0.599 / 0.401)."""
    l = np.array([[0.3, -1.2, 1.5, 2.0, -0.4, 1.6, 0.9, -2.1]], dtype=np.float32)
    s = moe.shape(1, 64, 8, 2, 64)
    ids = i32(2).view(1, 2)
    wt = torch.empty(1, 2, device="cuda")
    moe.moe_route_from_logits(s, torch.from_numpy(l).cuda(), ids, wt)
    torch.cuda.synchronize()
    assert ids.cpu().tolist() == [[3, 5]]
    assert np.round(wt.cpu().numpy()[0].astype(np.float64), 3).tolist() == [0.599, 0.401]


@pytest.mark.parametrize("sigma", [0.0, 1.0, 5.0])
def test_histogram_segments_and_plan_on_given_ids(sigma):
    E, R, S, k, B = 64, 4, 300, 4, 16
    T = R * S
    ids = syn.lognormal_topk_ids(E, T, k, sigma, seed=3)
    counts_ref = oracle.histogram(ids.numpy(), E)
    s = moe.shape(T, 64, E, k, 64, n_groups=R, replica_slots=B)
    counts = i32(E)
    moe.moe_histogram(s, ids.cuda(), counts)
    n_seg, rows = moe.moe_layout(s)
    se, so, sf = i32(n_seg), i32(n_seg + 1), i32(n_seg)
    st = i32(1)
    moe.moe_plan_balanced(s, counts, se, so, sf, st)
    torch.cuda.synchronize()
    assert (counts.cpu().numpy() == counts_ref).all()
    segs, _ = oracle.balanced_plan(counts_ref, R, S, k, B)
    assert st.item() == 0
    assert (se.cpu().numpy() == segs.expert).all()
    assert (so.cpu().numpy() == segs.offsets).all()
    assert (sf.cpu().numpy() == segs.first_rank).all()
    # plain segments with a capacity
    s2 = moe.shape(T, 64, E, k, 64, capacity=40)
    se2, so2, sf2 = i32(E), i32(E + 1), i32(E)
    moe.moe_segments(s2, counts, se2, so2, sf2)
    torch.cuda.synchronize()
    ref2 = oracle.plain_segments(counts_ref, 40)
    assert (so2.cpu().numpy() == ref2.offsets).all() and (se2.cpu().numpy() == ref2.expert).all()


@pytest.mark.parametrize("T,E,R", [(140000, 16, 4), (140032, 32, 32)], ids=["4-groups", "32-groups"])
def test_dispatch_large_balanced_plan(T, E, R):
    """A balanced plan with more than 2^20 pairs: with 4 groups the grouped dispatch (per-group
    counts, then every CTA ranking its own group's pairs), with 32 groups the multi-launch path
    (histogram partials, plan, look-back ranks, row copies): tables and positions bit for bit
    against the oracle."""
    d, k, B = 64, 8, 4
    ids = syn.lognormal_topk_ids(E, T, k, 1.0, seed=12).cuda()
    s = moe.shape(T, d, E, k, 64, n_groups=R, replica_slots=B)
    n_seg, rows = moe.moe_layout(s)
    disp, _ = moe.moe_workspace_size(s)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(13)).to(torch.bfloat16)
    counts, se, so, sf, dest, src = i32(E), i32(n_seg), i32(n_seg + 1), i32(n_seg), i32(T * k), i32(rows)
    xp = torch.zeros(rows, d, dtype=torch.bfloat16, device="cuda")
    st = i32(1)
    moe.moe_dispatch(s, x.cuda(), ids, 0, counts, se, so, sf, dest, src, xp, st,
                     torch.empty(disp, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    ids_np = ids.view(T, k).cpu().numpy()
    rc = oracle.histogram(ids_np, E)
    segs, _ = oracle.balanced_plan(rc, R, T // R, k, B)
    rdest, rsrc = oracle.dispatch_positions(ids_np, segs, E)
    assert st.item() == 0
    assert (counts.cpu().numpy() == rc).all()
    assert (se.cpu().numpy() == segs.expert).all() and (so.cpu().numpy() == segs.offsets).all()
    assert (sf.cpu().numpy() == segs.first_rank).all()
    assert (dest.cpu().numpy() == rdest).all()
    assert (src.cpu().numpy() == rsrc).all()
    assert torch.equal(xp.cpu(), x[torch.from_numpy(rsrc // k)])


def test_dispatch_with_given_plan_tables():
    """plan_ready = 1: the permutation alone, on counts and tables from the oracle."""
    E, R, S, k, B, d = 32, 4, 200, 4, 8, 128
    T = R * S
    ids = syn.lognormal_topk_ids(E, T, k, 2.0, seed=4)
    counts_ref = oracle.histogram(ids.numpy(), E)
    segs, _ = oracle.balanced_plan(counts_ref, R, S, k, B)
    dest_ref, src_ref = oracle.dispatch_positions(ids.numpy(), segs, E)
    x = torch.randn(T, d).to(torch.bfloat16)
    s = moe.shape(T, d, E, k, 64, n_groups=R, replica_slots=B)
    n_seg, rows = moe.moe_layout(s)
    ws = torch.empty(moe.moe_workspace_size(s)[0], dtype=torch.uint8, device="cuda")
    dest, src = i32(T * k), i32(rows)
    xp = torch.zeros(rows, d, dtype=torch.bfloat16, device="cuda")
    to_i32 = lambda a: torch.from_numpy(np.asarray(a, dtype=np.int32)).cuda()
    st = i32(1)
    moe.moe_dispatch(s, x.cuda(), ids.cuda(), 1, to_i32(counts_ref), to_i32(segs.expert), to_i32(segs.offsets),
                     to_i32(segs.first_rank), dest, src, xp, st, ws)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert (dest.cpu().numpy() == dest_ref).all()
    assert (src.cpu().numpy() == src_ref).all()
    assert (to_np(xp) == oracle.permute_rows(x, src_ref, k)).all()


def test_expert_ffn_on_given_rows():
    w = syn.Workload("ffn", T=400, d=256, E=5, k=2, F=384, zipf_s=1.0)
    case = make_case(w, seed=6)
    ref = oracle.layer_forward(case.x, case.w_r, case.bias, case.wg, case.wu, case.wd, w.k)
    s = moe_shape(w)
    n_seg, rows = moe.moe_layout(s)
    xp = torch.from_numpy(ref.xp.astype(np.float32)).to(torch.bfloat16).cuda()
    to_i32 = lambda a: torch.from_numpy(np.asarray(a, dtype=np.int32)).cuda()
    hp = torch.empty(rows, w.F, dtype=torch.bfloat16, device="cuda")
    yp = torch.empty(rows, w.d, dtype=torch.float32, device="cuda")
    st = i32(1)
    moe.moe_expert_ffn(s, xp, to_i32(ref.segs.expert), to_i32(ref.segs.offsets), dev(case.wg), dev(case.wu),
                       dev(case.wd), hp, yp, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    check_bf16_storage(to_np(hp), ref.hp, "Hp")
    check_close(to_np(yp), ref.yp, "Yp")


def test_combine_on_given_rows():
    T, k, d, E = 300, 4, 192, 8
    ids = syn.lognormal_topk_ids(E, T, k, 1.0, seed=7).numpy()
    counts = oracle.histogram(ids, E)
    segs = oracle.plain_segments(counts, 120)     # drops some pairs
    dest, src = oracle.dispatch_positions(ids, segs, E)
    rows = int(segs.offsets[-1])
    yp = torch.randn(rows, d)
    wts = torch.rand(T, k)
    ref = oracle.combine(oracle.f64(yp), dest, oracle.f64(wts), T, k)
    s = moe.shape(T, d, E, k, 64, capacity=120)
    out = torch.empty(T, d, dtype=torch.float32, device="cuda")
    moe.moe_combine(s, yp.cuda(), torch.from_numpy(dest.astype(np.int32)).cuda(), wts.cuda(), out)
    torch.cuda.synchronize()
    # only fp32 accumulation (k terms) separates the two
    check_close(to_np(out), ref, "out", max_abs_of_rms=1e-5, mean_rel=1e-6)
    dropped_all = (dest.reshape(T, k) < 0).all(axis=1)
    assert (to_np(out)[dropped_all] == 0).all()


def test_infeasible_plan_reports_and_moves_nothing():
    w = syn.Workload("infeasible", T=256, d=64, E=8, k=1, F=64, zipf_s=3.0, n_groups=4, replica_slots=0)
    case = make_case(w, seed=8)
    got = run_layer(case)
    assert got["status"] & moe.DEV_ERR_PLAN
    assert (got["dest"].numpy() == -1).all()
    assert (got["seg_offsets"].numpy() == 0).all()
    assert (to_np(got["out"]) == 0).all()
    with pytest.raises(oracle.PlanInfeasible):
        oracle.balanced_plan(oracle.histogram(got["ids"].numpy(), 8), 4, 64, 1, 0)


def test_zero_tokens_is_a_no_op():
    s = moe.shape(0, 128, 8, 2, 256)
    ws = torch.empty(max(moe.moe_workspace_size(s)[1], 256), dtype=torch.uint8, device="cuda")
    dummy = torch.zeros(256, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(256, dtype=torch.float32, device="cuda")
    moe.moe_layer_fwd(s, dummy, dummy, None, dummy, dummy, dummy, out, None, ws)
    torch.cuda.synchronize()


def test_repeated_calls_are_deterministic():
    case = make_case(SMALL[1], seed=9)
    a = run_layer(case)
    b = run_layer(case)
    assert torch.equal(a["out"], b["out"]) and torch.equal(a["dest"], b["dest"])
    assert torch.equal(a["hp"], b["hp"])


def _shared_case(seed=10):
    w = syn.Workload("shared", T=333, d=192, E=6, k=2, F=128, zipf_s=1.0)
    case = make_case(w, seed=seed)
    Fs = 320
    gs, us, ds = syn.shared_expert_weights(w, Fs, seed)
    return w, case, Fs, (gs, us, ds)


def test_shared_expert_and_combine_add():
    """Shared expert (dense SwiGLU on every token) and the combine with a base term."""
    w, case, Fs, sh = _shared_case()
    ref = oracle.layer_forward(case.x, case.w_r, case.bias, case.wg, case.wu, case.wd, w.k, shared=sh)
    s = moe_shape(w)
    h_s = torch.empty(w.T, Fs, dtype=torch.bfloat16, device="cuda")
    y_s = torch.empty(w.T, w.d, dtype=torch.float32, device="cuda")
    st = i32(1)
    moe.moe_shared_expert(s, Fs, dev(case.x), *(dev(t) for t in sh), h_s, y_s, st)
    got = run_layer(case)
    out = torch.empty(w.T, w.d, dtype=torch.float32, device="cuda")
    v = moe.moe_layer_views(s, got["ws"])
    base = got["ws"].data_ptr()
    n_seg, rows = moe.moe_layout(s)
    yp = got["yp"]
    dest = got["ws"][v.dest - base:][: w.T * w.k * 4].view(torch.int32)
    tw = got["ws"][v.topk_w - base:][: w.T * w.k * 4].view(torch.float32)
    moe.moe_combine_add(s, yp, dest, tw, y_s, out)
    torch.cuda.synchronize()
    assert st.item() == 0
    check_close(to_np(y_s), oracle.shared_expert(case.x, *sh), "shared expert")
    check_close(to_np(out), ref.out, "routed + shared")
    # base = None is exactly moe_combine
    out2 = torch.empty_like(out)
    moe.moe_combine_add(s, yp, dest, tw, None, out2)
    torch.cuda.synchronize()
    assert torch.equal(out2, got["out"])


@pytest.mark.parametrize("T", [270, 128, 97])
def test_shared_expert_row_tails(T):
    """The shared expert's down projection over T rows whose last 128-row tile holds 14, 128 or 97
    rows (14 takes the swapped-operand tail of the down projection; d = 512 gives it full 256-column
    weight tiles)."""
    w = syn.Workload("shared-tail", T=T, d=512, E=4, k=2, F=128)
    case = make_case(w, seed=12)
    Fs = 320
    sh = syn.shared_expert_weights(w, Fs, 12)
    s = moe_shape(w)
    h_s = torch.empty(w.T, Fs, dtype=torch.bfloat16, device="cuda")
    y_s = torch.empty(w.T, w.d, dtype=torch.float32, device="cuda")
    st = i32(1)
    moe.moe_shared_expert(s, Fs, dev(case.x), *(dev(t) for t in sh), h_s, y_s, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    check_close(to_np(y_s), oracle.shared_expert(case.x, *sh), "shared expert")


def test_shared_expert_overlapped_on_a_second_stream():
    """Run on a side stream while the routed path runs; joined by an event, the result is bit-identical."""
    w, case, Fs, sh = _shared_case(seed=11)
    s = moe_shape(w)
    x = dev(case.x)
    shd = [dev(t) for t in sh]
    h1 = torch.empty(w.T, Fs, dtype=torch.bfloat16, device="cuda")
    y1 = torch.empty(w.T, w.d, dtype=torch.float32, device="cuda")
    moe.moe_shared_expert(s, Fs, x, *shd, h1, y1)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    start = torch.cuda.Event()
    start.record()
    side.wait_event(start)
    h2 = torch.empty_like(h1)
    y2 = torch.full_like(y1, float("nan"))
    moe.moe_shared_expert(s, Fs, x, *shd, h2, y2, stream=side)
    got = run_layer(case)                       # the routed path on the default stream meanwhile
    done = torch.cuda.Event()
    done.record(side)
    torch.cuda.current_stream().wait_event(done)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


GRAPHED = [
    SMALL[1],  # ragged top-k, single-pass router
    syn.Workload("split-router", T=600, d=1024, E=16, k=2, F=128, zipf_s=0.8),  # router split over CTAs
    syn.Workload("plan", T=512, d=128, E=16, k=4, F=128, zipf_s=1.2, n_groups=4, replica_slots=8),
    syn.Workload("lookback", T=9000, d=64, E=64, k=8, F=64, zipf_s=0.5),  # memset + look-back dispatch
    syn.Workload("reroute", T=300, d=128, E=8, k=2, F=192, zipf_s=1.2, capacity_factor=0.9, reroute=True),
    syn.Workload("expert-choice", T=700, d=128, E=8, k=2, F=192, zipf_s=1.0, capacity_factor=1.0,
                 expert_choice=True),
]


@pytest.mark.parametrize("w", GRAPHED, ids=[w.name for w in GRAPHED])
def test_layer_fwd_captured_in_a_cuda_graph(w):
    """The whole layer allocates nothing and never synchronises, so it can be captured into a
    CUDA graph and replayed; replays read the same device buffers and match eager calls.  Every
    dispatch mode: the count kernel, the balanced plan, the look-back (with its memset), the
    re-routing rounds (a cooperative launch) and expert choice."""
    case = make_case(w, seed=14)
    s = moe_shape(w)
    _, layer_bytes = moe.moe_workspace_size(s)
    ws = torch.empty(layer_bytes, dtype=torch.uint8, device="cuda")
    x, w_r, bias = dev(case.x), dev(case.w_r), dev(case.bias)
    wg, wu, wd = dev(case.wg), dev(case.wu), dev(case.wd)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    eager = torch.empty(w.T, w.d, dtype=torch.float32, device="cuda")
    moe.moe_layer_fwd(s, x, w_r, bias, wg, wu, wd, eager, status, ws)   # warm-up outside capture
    torch.cuda.synchronize()

    graphed = torch.zeros_like(eager)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_layer_fwd(s, x, w_r, bias, wg, wu, wd, graphed, status, ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(graphed, eager)

    # new input values in the same buffer: the replay follows them
    x.copy_(dev(syn.router_inputs(w, 99)[0]))
    g.replay()
    moe.moe_layer_fwd(s, x, w_r, bias, wg, wu, wd, eager, status, ws)
    torch.cuda.synchronize()
    assert torch.equal(graphed, eager)
    assert status.item() == 0


@pytest.mark.parametrize("name", ["capacity", "plan"])
def test_layer_fwd_aux_copies_the_routing_results(name):
    """moe_layer_fwd_aux: the same output as moe_layer_fwd, and the routing results (ids, weights,
    counts, segment offsets, dest, statistics) in the caller's buffers equal the oracle's."""
    w = next(x for x in SMALL if x.name == name)
    case = make_case(w, seed=1)
    ref = _oracle_layer(case)
    s = moe_shape(w)
    s.out_dtype = moe.DTYPE_BF16
    n_seg, rows = moe.moe_layout(s)
    ws = torch.empty(moe.moe_workspace_size(s)[1], dtype=torch.uint8, device="cuda")
    out = torch.empty(w.T, w.d, dtype=torch.bfloat16, device="cuda")
    st = i32(1)
    ids, wts = i32(w.T * w.k), torch.zeros(w.T * w.k, device="cuda")
    counts, offs, dest, stats = i32(w.E), i32(n_seg + 1), i32(w.T * w.k), i32(len(moe.STAT_NAMES))
    moe.moe_layer_fwd_aux(s, dev(case.x), dev(case.w_r), dev(case.bias), dev(case.wg), dev(case.wu), dev(case.wd),
                          out, st, ws, topk_ids=ids, topk_w=wts, counts=counts, seg_offsets=offs, dest=dest,
                          stats=stats)
    torch.cuda.synchronize()
    assert st.item() == 0
    plain = run_layer(case, out_dtype=moe.DTYPE_BF16)
    assert torch.equal(out, plain["out"])
    assert (ids.cpu().numpy().reshape(w.T, w.k) == ref.ids).all()
    assert np.abs(wts.cpu().numpy().reshape(w.T, w.k) - ref.weights).max() < 1e-4
    assert (counts.cpu().numpy() == ref.counts).all()
    assert (offs.cpu().numpy() == ref.segs.offsets).all()
    assert (dest.cpu().numpy() == ref.dest).all()
    got = dict(zip(moe.STAT_NAMES, stats.cpu().tolist()))
    assert got["pairs"] == w.T * w.k and got["rows"] == int(ref.segs.offsets[-1])
    assert got["dropped"] == int((ref.dest < 0).sum()) and got["max_expert_load"] == int(ref.counts.max())
