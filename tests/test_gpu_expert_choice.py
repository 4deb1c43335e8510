"""Expert-choice routing on the GPU against the oracle ("Expert를 똑같이 나눴는데도 GPU가
대기하는 이유: MoE의 토큰 쏠림", section "라우팅 분포와 학습 안정성": experts choose
tokens instead of tokens choosing experts).

The selection is compared bit for bit (picked tokens, their rows, the row map, the segment
table, the dispatched rows); the scores and row weights within fp32 rounding; Hp, Yp and the
output with the same tolerances as the top-k path.  The inputs keep every expert's C-th and
(C+1)-th scores at least 5e-4 (relative) apart, so the fp32 scores of both sides select the same
tokens.
"""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

from gpu_cases import capacity_rows, check_bf16_storage, check_close, expert_rows, make_case, run_layer, to_np

pytestmark = pytest.mark.gpu

W = syn.Workload
SMALL = [
    W("ec-small", T=300, d=128, E=8, k=2, F=192, capacity_factor=1.0, expert_choice=True),        # C = 75
    W("ec-chunks", T=2500, d=256, E=12, k=1, F=256, capacity_factor=2.0, expert_choice=True),     # 3 scan chunks
    W("ec-cap-above-T", T=50, d=64, E=4, k=2, F=64, capacity_factor=3.0, expert_choice=True),     # C = 75 > T
    W("ec-e256", T=520, d=128, E=256, k=4, F=128, zipf_s=1.2, capacity_factor=1.0, expert_choice=True),  # C = 9
    W("ec-one-token", T=1, d=64, E=3, k=1, F=64, capacity_factor=1.0, expert_choice=True),
]


def _check_scores(got, ref):
    """fp32 softmax of fp32 logits (tensor-core sums over d): relative error about the logits' absolute error,
    measured up to 3.4e-5 at d = 4096."""
    assert (np.abs(got - ref) <= 1e-4 * ref + 1e-9).all(), float(np.abs(got / ref - 1).max())


def _check_selection(got, ec, T, E):
    assert (got["seg_expert"].numpy() == np.arange(E)).all()
    assert (got["seg_offsets"].numpy() == ec.segs.offsets).all()
    assert (got["src"].numpy() == ec.src).all(), "picked tokens differ"
    assert (got["emap"].numpy() == oracle.expert_choice_map(ec, T)).all(), "row map differs"
    if len(ec.src):
        assert (np.abs(got["row_w"].numpy() - ec.row_w) <= 1e-4 * np.abs(ec.row_w) + 1e-9).all()


def _check_elementwise(got, ref, bound, what):
    """|got - ref| <= bound (+ a tiny absolute term) and mean-rel <= 5e-3.  The bound is
    2^-7 * sum over the token's rows of |w| * (|h| . |W_d[e]|^T): one bf16 ulp of Hp, the
    operand of the down projection, carried to the output (it covers the fp32 sums too).
    Unlike max-abs <= 2e-2 * RMS it holds for heavy-tailed outputs (a Zipf router bias gives
    some tokens many experts and others none)."""
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    bad = err > bound + 1e-7 * max(rms, 1e-30)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert not bad.any(), f"{what}: {int(bad.sum())} elements above the bound"
    denom = float(np.abs(ref).sum())
    if denom > 0:
        assert float(err.sum()) / denom <= 5e-3, f"{what}: mean-rel {float(err.sum()) / denom:.3e}"


def _check_output(got_out, ref_out, ec, hp, wd, what="out"):
    T = ref_out.shape[0]
    chosen = np.zeros(T, dtype=bool)
    chosen[np.asarray(ec.src, dtype=np.int64)] = True
    assert (got_out[~chosen] == 0).all(), f"{what}: tokens no expert kept are not zero"
    a = np.zeros((hp.shape[0], ref_out.shape[1]))
    off = ec.segs.offsets
    for e in range(len(ec.picks)):
        if off[e + 1] > off[e]:
            a[off[e]:off[e + 1]] = np.abs(hp[off[e]:off[e + 1]]) @ np.abs(oracle.f64(wd[e])).T
    bound = 2.0 ** -7 * oracle.combine_expert_choice(a, ec.src, np.abs(ec.row_w), T)
    _check_elementwise(got_out, ref_out, bound, what)


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_expert_choice_layer_matches_oracle(cuda_ok, w):
    case = make_case(w, seed=5)
    C = capacity_rows(w)
    logits, ec, xp, hp, yp, out = oracle.expert_choice_forward(case.x, case.w_r, case.bias, case.wg, case.wu,
                                                                case.wd, C)
    got = run_layer(case)
    assert got["status"] == 0
    assert got["rows"] == w.E * min(C, w.T)
    _check_scores(got["scores"].numpy().T, ec.scores)
    _check_selection(got, ec, w.T, w.E)
    assert (to_np(got["xp"]) == xp).all()
    check_bf16_storage(to_np(got["hp"]), hp, "Hp")
    check_close(to_np(got["yp"]), yp, "Yp")
    _check_output(to_np(got["out"]), out, ec, hp, case.wd)
    if w.zipf_s == 0:   # outputs of one scale: the layer tolerance (max-abs <= 2e-2 RMS) holds as well
        kept = (oracle.expert_choice_map(ec, w.T) >= 0).any(axis=1)
        check_close(to_np(got["out"])[kept], out[kept], "out")


@pytest.mark.parametrize("T,E,C", [(3000, 5, 700), (50000, 3, 9000)])
def test_selection_with_many_equal_scores(cuda_ok, T, E, C):
    """Scores on a coarse grid (many equal values at every threshold) and of both signs:
    equal scores go to the lower token id; the whole selection is bit-exact.  The larger case
    has more tokens than the selection keeps in shared memory (it reads the scores from global
    memory in every pass)."""
    d = 64
    rng = np.random.default_rng(7)
    S = (rng.integers(-3, 6, size=(T, E)) / 8.0).astype(np.float32)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16)
    s = moe.shape(T, d, E, 1, 64, capacity=C, route_flags=moe.ROUTE_EXPERT_CHOICE)
    n_seg, rows = moe.moe_layout(s)
    assert (n_seg, rows) == (E, E * C)
    z = lambda n, dt=torch.int32: torch.full((n,), -7, dtype=dt, device="cuda")
    seg_expert, seg_offsets, src, emap = z(E), z(E + 1), z(rows), z(T * E)
    row_w = z(rows, torch.float32)
    xp = torch.zeros(rows, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_choose(s, torch.from_numpy(np.ascontiguousarray(S.T)).cuda(), x.cuda(), seg_expert, seg_offsets,
                          src, row_w, emap, xp)
    torch.cuda.synchronize()
    ec = oracle.select_tokens(S, C)
    got = dict(seg_expert=seg_expert.cpu(), seg_offsets=seg_offsets.cpu(), src=src.cpu(), row_w=row_w.cpu(),
               emap=emap.view(T, E).cpu())
    _check_selection(got, ec, T, E)
    assert (row_w.cpu().numpy() == S[ec.src, np.repeat(np.arange(E), C)]).all()
    assert torch.equal(xp.cpu(), x[torch.from_numpy(ec.src)])


def test_combine_with_base(cuda_ok):
    """moe_combine_expert_choice adds onto a base (e.g. a shared expert's output); out may alias it."""
    T, E, C, d = 700, 6, 150, 128
    rng = np.random.default_rng(9)
    ec = oracle.select_tokens(rng.random((T, E)), C)
    rows = E * C
    yp = rng.normal(size=(rows, d)).astype(np.float32)
    base = rng.normal(size=(T, d)).astype(np.float32)
    s = moe.shape(T, d, E, 1, 64, capacity=C, route_flags=moe.ROUTE_EXPERT_CHOICE)
    emap = torch.from_numpy(oracle.expert_choice_map(ec, T).astype(np.int32)).cuda()
    row_w = torch.from_numpy(ec.row_w.astype(np.float32)).cuda()
    out = torch.from_numpy(base).cuda()
    moe.moe_combine_expert_choice(s, torch.from_numpy(yp).cuda(), emap, row_w, out, out)
    torch.cuda.synchronize()
    ref = base + oracle.combine_expert_choice(yp, ec.src, ec.row_w.astype(np.float32), T)
    assert np.abs(out.cpu().numpy() - ref).max() < 1e-5 * max(1.0, np.abs(ref).max())


def test_deterministic(cuda_ok):
    case = make_case(SMALL[1], seed=11)
    a, b = run_layer(case), run_layer(case)
    assert torch.equal(a["out"], b["out"])


def test_calls_reject_the_other_routing(cuda_ok):
    ec = moe.shape(64, 128, 8, 2, 128, capacity=16, route_flags=moe.ROUTE_EXPERT_CHOICE)
    topk = moe.shape(64, 128, 8, 2, 128)
    dummy = torch.zeros(1 << 16, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.moe_route(ec, dummy, dummy, None, None, dummy, dummy, dummy)
    with pytest.raises(moe.MoeError):
        moe.moe_combine(ec, dummy, dummy, dummy, dummy)
    with pytest.raises(moe.MoeError):
        moe.moe_route_scores(topk, dummy, dummy, None, dummy)
    with pytest.raises(moe.MoeError):
        moe.moe_combine_expert_choice(topk, dummy, dummy, dummy, None, dummy)


FULL = [syn.EXPERT_CHOICE, syn.EXPERT_CHOICE_E64]


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_full_size_expert_choice(cuda_ok, w):
    """The benchmark's expert-choice workloads at full size through moe_layer_fwd: the whole
    selection bit for bit; Hp / Yp on sampled rows and the output on sampled tokens in fp64."""
    case = make_case(w, seed=0, weights_device="cuda")
    C = capacity_rows(w)
    got = run_layer(case)
    assert got["status"] == 0
    ec = oracle.expert_choice(oracle.router_logits(case.x, case.w_r, case.bias), C)
    _check_scores(got["scores"].numpy().T, ec.scores)
    _check_selection(got, ec, w.T, w.E)
    src_dev = torch.from_numpy(ec.src.astype(np.int64)).cuda()
    assert torch.equal(got["xp"], got["x_dev"][src_dev])

    rng = np.random.default_rng(0)
    x64 = oracle.f64(case.x)
    experts = sorted(set(rng.choice(w.E, size=min(8, w.E), replace=False).tolist()))
    rows = []
    for e in experts:
        a, b = int(ec.segs.offsets[e]), int(ec.segs.offsets[e + 1])
        rows += sorted({a, b - 1, (a + b) // 2})
    emap = oracle.expert_choice_map(ec, w.T)
    toks = sorted(set(rng.choice(w.T, size=12, replace=False).tolist()) | {0, w.T - 1})
    row_e = {r: int(np.searchsorted(ec.segs.offsets, r, side="right") - 1) for r in rows}
    pairs = [(("row", r), x64[ec.src[r]], row_e[r]) for r in rows]
    pairs += [(("tok", t, e), x64[t], e) for t in toks for e in range(w.E) if emap[t, e] >= 0]
    ref = expert_rows(pairs, case.wg, case.wu, case.wd, with_bound=True)

    rsel = torch.tensor(rows, device="cuda")
    check_bf16_storage(to_np(got["hp"][rsel]), np.stack([ref[("row", r)][0] for r in rows]), "Hp (sampled rows)")
    check_close(to_np(got["yp"][rsel]), np.stack([ref[("row", r)][1] for r in rows]), "Yp (sampled rows)")

    ref_out = np.zeros((len(toks), w.d))
    bound = np.zeros((len(toks), w.d))
    for i, t in enumerate(toks):
        for e in range(w.E):
            if emap[t, e] >= 0:
                _, y, a = ref[("tok", t, e)]
                ref_out[i] += ec.scores[t, e] * y
                bound[i] += ec.scores[t, e] * a
    got_out = to_np(got["out"][torch.tensor(toks, device="cuda")])
    kept = (emap[toks] >= 0).any(axis=1)
    assert (got_out[~kept] == 0).all()
    _check_elementwise(got_out, ref_out, 2.0 ** -7 * bound, "out (sampled tokens)")
    if w.zipf_s == 0:
        check_close(got_out[kept], ref_out[kept], "out (sampled tokens)")
