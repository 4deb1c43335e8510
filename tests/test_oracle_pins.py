"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: each check uses a value the
pages print, a closed form, brute force, an independent library routine or
an invariant.  ``test_planted_mistakes_are_caught`` plants plausible bugs in
the oracle (on the CPU) and shows that one of these pins fails for each.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import moe_oracle as om
from mixture_experts_routing_02_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            out[key.strip()] = val.split()
    return out


# --------------------------------------------------------------------------- pins as functions
# (returning True when the pin holds, so the planted-mistake test can reuse them)

def pin_worked_example():
    g = _read_golden("worked_top2.txt")
    logits = np.array([[float(v) for v in g["logits"]]])
    k = int(g["k"][0])
    ids = oracle.topk_ids(logits, k)
    w = oracle.topk_weights(logits, ids)
    ok = list(ids[0]) == [int(v) for v in g["ids"]]
    ok &= np.allclose(np.round(w[0], 3), [float(v) for v in g["weights_3dp"]], atol=0, rtol=0)
    closed = math.exp(0.4) / (1 + math.exp(0.4))
    ok &= abs(w[0, 0] - closed) < 1e-12 and abs(w[0, 1] - (1 - closed)) < 1e-12
    return bool(ok)


def pin_topk_brute_force(seed=0, T=40, E=7):
    rng = np.random.default_rng(seed)
    logits = rng.normal(size=(T, E))
    for k in range(1, E + 1):
        ids = oracle.topk_ids(logits, k)
        for t in range(T):
            l32 = logits[t].astype(np.float32).astype(np.float64)
            best = max(itertools.combinations(range(E), k), key=lambda s: sum(l32[list(s)]))
            want = sorted(best, key=lambda e: -l32[e])
            if list(ids[t]) != want:
                return False
    return True


def pin_weights_full_softmax(seed=1, T=50, E=16, k=4):
    rng = np.random.default_rng(seed)
    logits = rng.normal(scale=3.0, size=(T, E))
    ids = oracle.topk_ids(logits, k)
    w = oracle.topk_weights(logits, ids)
    p = torch.softmax(torch.from_numpy(logits), dim=1).numpy()
    sel = np.take_along_axis(p, ids, axis=1)
    ref = sel / sel.sum(axis=1, keepdims=True)
    return bool(np.allclose(w, ref, rtol=1e-12, atol=1e-15)
                and np.allclose(w.sum(1), 1.0, atol=1e-14)
                and (np.diff(w, axis=1) <= 0).all())


def pin_weights_softmax_all(seed=12, T=40, E=12, k=3):
    """Softmax over all E (library softmax), read at the selected experts, no renormalisation."""
    rng = np.random.default_rng(seed)
    logits = rng.normal(scale=2.0, size=(T, E))
    ids = oracle.topk_ids(logits, k)
    w = oracle.topk_weights_softmax_all(logits, ids)
    p = torch.softmax(torch.from_numpy(logits), dim=1).numpy()
    ref = np.take_along_axis(p, ids, axis=1)
    return bool(np.allclose(w, ref, rtol=1e-12, atol=1e-15) and (w.sum(1) < 1).all()
                and np.allclose(w / w.sum(1, keepdims=True), oracle.topk_weights(logits, ids), rtol=1e-12))


def pin_router_logits_library(seed=2):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(37, 96, generator=g).to(torch.bfloat16)
    wr = (torch.randn(11, 96, generator=g) * 0.02).to(torch.bfloat16)
    b = torch.randn(11, generator=g)
    ref = torch.nn.functional.linear(x.double(), wr.double(), b.double()).numpy()
    return bool(np.allclose(oracle.router_logits(x, wr, b), ref, rtol=1e-13, atol=1e-13))


def pin_histogram_bincount(seed=3, T=300, E=13, k=3):
    ids = syn.lognormal_topk_ids(E, T, k, 1.0, seed=seed).numpy()
    c = oracle.histogram(ids, E)
    return bool(c.sum() == T * k and (c == np.bincount(ids.ravel(), minlength=E)).all())


def pin_rank_stable_sort(seed=4, T=200, E=9, k=3):
    ids = syn.lognormal_topk_ids(E, T, k, 1.5, seed=seed).numpy()
    flat = ids.ravel()
    rank = oracle.expert_rank(ids, E)
    order = np.argsort(flat, kind="stable")
    first = np.searchsorted(flat[order], np.arange(E))
    want = np.empty_like(rank)
    want[order] = np.arange(flat.size) - first[flat[order]]
    return bool((rank == want).all())


def _small_layer(seed, T=24, d=64, E=6, k=2, F=64, zipf=0.0):
    w = syn.Workload("pin", T=T, d=d, E=E, k=k, F=F, zipf_s=zipf)
    x, wr, b = syn.router_inputs(w, seed)
    oracle.enforce_margin(x, wr, b, k, lambda t, a: syn.x_row_redraw(w, seed, t, a))
    wg, wu, wd = syn.expert_weights(w, seed)
    return x, wr, b, wg, wu, wd


def pin_layer_equals_eager(seed=5, capacity=0):
    """The dispatched layer equals a per-token, per-expert loop (the 'eager' backend)."""
    T, E, k = 24, 6, 2
    x, wr, b, wg, wu, wd = _small_layer(seed, T=T, E=E, k=k, zipf=1.2)
    res = oracle.layer_forward(x, wr, b, wg, wu, wd, k, capacity=capacity)
    x64 = oracle.f64(x)
    logits = oracle.router_logits(x, wr, b)
    seen = {}
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-np.float32(logits[t, e]), e))[:k]
        sel = logits[t, order]
        w = np.exp(sel - sel.max()); w /= w.sum()
        keep = []
        for e in order:
            seen[e] = seen.get(e, 0) + 1
            keep.append(capacity == 0 or seen[e] <= capacity)
        want = oracle.token_output(x64[t], order, w, wg, wu, wd, keep=keep)
        if not np.allclose(res.out[t], want, rtol=1e-11, atol=1e-13):
            return False
    return True


def pin_dense_ffn_e1k1(seed=6):
    """E = 1, k = 1 reduces to one dense SwiGLU FFN applied to every token."""
    x, wr, b, wg, wu, wd = _small_layer(seed, T=17, E=1, k=1)
    res = oracle.layer_forward(x, wr, b, wg, wu, wd, 1)
    F_ = torch.nn.functional
    xd = x.double()
    ref = F_.linear(F_.silu(F_.linear(xd, wg[0].double())) * F_.linear(xd, wu[0].double()),
                    wd[0].double()).numpy()
    return bool(np.allclose(res.out, ref, rtol=1e-11, atol=1e-13))


def pin_shared_expert_additive(seed=8):
    """With a shared expert the output is the routed output plus a dense SwiGLU FFN (library linear/silu)."""
    T, E, k, Fs = 20, 6, 2, 96
    x, wr, b, wg, wu, wd = _small_layer(seed, T=T, E=E, k=k)
    w = syn.Workload("pin", T=T, d=64, E=E, k=k, F=64)
    gs, us, ds = syn.shared_expert_weights(w, Fs, seed)
    routed = oracle.layer_forward(x, wr, b, wg, wu, wd, k).out
    both = oracle.layer_forward(x, wr, b, wg, wu, wd, k, shared=(gs, us, ds)).out
    F_ = torch.nn.functional
    xd = x.double()
    dense = F_.linear(F_.silu(F_.linear(xd, gs.double())) * F_.linear(xd, us.double()), ds.double()).numpy()
    return bool(np.allclose(both - routed, dense, rtol=1e-10, atol=1e-13))


def pin_expert_choice_brute_force(seed=20, T=7, E=3, C=3):
    """Each expert's picks are the C-subset of tokens with the largest summed scores (brute force),
    listed in ascending id; scores are the library softmax over experts."""
    rng = np.random.default_rng(seed)
    logits = rng.normal(size=(T, E))
    ec = oracle.expert_choice(logits, C)
    S = torch.softmax(torch.from_numpy(logits), dim=1).numpy()
    ok = np.allclose(ec.scores, S, rtol=1e-12, atol=1e-15)
    for e in range(E):
        s32 = S[:, e].astype(np.float32).astype(np.float64)
        best = max(itertools.combinations(range(T), C), key=lambda sub: sum(s32[list(sub)]))
        ok &= list(ec.picks[e]) == sorted(best)
    ok &= (ec.segs.offsets == np.arange(E + 1) * C).all()
    return bool(ok)


def pin_expert_choice_layer_eager(seed=21):
    """The expert-choice layer equals a per-expert loop over its picked tokens."""
    T, E, C = 30, 4, 9
    x, wr, b, wg, wu, wd = _small_layer(seed, T=T, E=E, k=1)
    logits, ec, xp, hp, yp, out = oracle.expert_choice_forward(x, wr, b, wg, wu, wd, C)
    x64 = oracle.f64(x)
    S = oracle.expert_scores(oracle.router_logits(x, wr, b))
    want = np.zeros_like(out)
    for e in range(E):
        s32 = S[:, e].astype(np.float32)
        chosen = sorted(range(T), key=lambda t: (-s32[t], t))[:C]
        for t in chosen:
            _, y = oracle.expert_ffn(x64[t][None, :], wg[e], wu[e], wd[e])
            want[t] += S[t, e] * y[0]
    return bool(np.allclose(out, want, rtol=1e-11, atol=1e-13))


def pin_reroute_worked_example():
    """Hand-worked: C = 1, k = 1, E = 3; tokens 0-2 rank the experts 0 > 1 > 2, token 3 ranks
    0 > 2 > 1; everyone picks expert 0.  Round 0: token 0 keeps expert 0.  Round 1 (experts 1, 2
    open): tokens 1 and 2 propose 1, token 3 proposes 2; expert 1 takes token 1 (q order).
    Round 2: no expert has room, token 2 is dropped."""
    l = np.array([[3, 2, 1], [3, 2, 1], [3, 2, 1], [3, 1, 2]], dtype=np.float64)
    rr = oracle.reroute_overflow(np.zeros((4, 1), dtype=np.int64), l, 1)
    return (list(rr.expert) == [0, 1, -1, 2] and list(rr.slot) == [0, 0, -1, 0] and list(rr.round) == [0, 1, -1, 1]
            and list(rr.assigned) == [1, 1, 1])


def pin_reroute_without_overflow(seed=30):
    """With room for every pair the re-routing is the plain top-k dispatch (library argsort ranks)."""
    rng = np.random.default_rng(seed)
    T, E, k = 50, 6, 2
    logits = rng.normal(size=(T, E))
    ids = oracle.topk_ids(logits, k)
    rr = oracle.reroute_overflow(ids, logits, T * k)
    flat = ids.ravel()
    rank = np.empty(T * k, dtype=np.int64)
    for e in range(E):
        qs = np.nonzero(flat == e)[0]                 # ascending q: the stable order
        rank[qs] = np.arange(len(qs))
    return bool((rr.expert == flat).all() and (rr.slot == rank).all() and (rr.round == 0).all())


def pin_reroute_invariants(seed=31):
    """Random skewed cases: no expert over C; a token never holds an expert twice; a moved pair
    sits at an expert below the token's top-k, and a token's moved pairs follow its logit order
    (j order); a pair is dropped only when every expert its token does not hold is full; slots of
    each expert are 0..assigned-1 with round-major, q-minor order."""
    rng = np.random.default_rng(seed)
    ok = True
    for trial in range(6):
        T, E, k = 40, 7, 2
        logits = rng.normal(size=(T, E)) + np.linspace(2, 0, E)[None, :]   # skew toward low ids
        ids = oracle.topk_ids(logits, k)
        C = int(rng.integers(2, 9))
        rr = oracle.reroute_overflow(ids, logits, C)
        ok &= bool((rr.assigned <= C).all())
        for t in range(T):
            fin = [int(e) for e in rr.expert[t * k:(t + 1) * k] if e >= 0]
            ok &= len(set(fin)) == len(fin)
            order = [e for e in oracle.candidate_order(logits[t].astype(np.float32)) if e not in ids[t]]
            moved = [int(rr.expert[t * k + j]) for j in range(k) if rr.round[t * k + j] > 0]
            ok &= all(e in order for e in moved)
            ok &= [order.index(e) for e in moved] == sorted(order.index(e) for e in moved)
            if (rr.expert[t * k:(t + 1) * k] < 0).any():
                others = [e for e in range(E) if e not in fin]
                ok &= all(rr.assigned[e] == C for e in others)
        for e in range(E):
            qs = np.nonzero(rr.expert == e)[0]
            ok &= sorted(rr.slot[qs].tolist()) == list(range(len(qs)))
            keyed = sorted(qs.tolist(), key=lambda q: (rr.round[q], q))
            ok &= [int(rr.slot[q]) for q in keyed] == list(range(len(qs)))
        ok &= int((rr.expert >= 0).sum()) == int(rr.assigned.sum())
    return bool(ok)


def pin_reroute_positions_worked():
    """Hand-worked layout of a re-routed result: T = 4 tokens, k = 2, E = 3.  Final experts per
    pair q = t*k + j: [1, 0, 0, 2, 1, -, 2, 1] with slots inside each expert
    [0, 0, 1, 0, 1, -, 1, 2]; so the experts hold 2, 3 and 2 rows, the segments start at rows
    0, 2, 5 (7 rows in all), dest[q] = start of its expert + slot = [2, 0, 1, 5, 3, -1, 6, 4] and
    the inverse src[row] = [1, 2, 0, 4, 7, 3, 6]."""
    rr = om.Rerouted(expert=np.array([1, 0, 0, 2, 1, -1, 2, 1]), slot=np.array([0, 0, 1, 0, 1, -1, 1, 2]),
                     round=np.array([0, 0, 0, 0, 0, -1, 1, 1]), assigned=np.array([2, 3, 2]))
    segs, dest, src = oracle.reroute_positions(rr)
    return bool(list(segs.offsets) == [0, 2, 5, 7] and list(segs.expert) == [0, 1, 2]
                and list(dest) == [2, 0, 1, 5, 3, -1, 6, 4] and list(src) == [1, 2, 0, 4, 7, 3, 6])


def pin_layer_reroute_eager(seed=32):
    """The re-routed layer equals an eager loop over the pairs: pair (t, j) placed at expert
    e = rr.expert[q] adds w[t, j] * FFN_e(x_t) to token t (a moved pair keeps its routing weight;
    a dropped pair adds nothing), and the dispatched row of every placed pair is x_t."""
    T, E, k, C = 40, 6, 2, 8
    x, wr, b, wg, wu, wd = _small_layer(seed, T=T, E=E, k=k, zipf=1.5)
    logits, ids, w, rr, segs, dest, src, xp, hp, yp, out = oracle.layer_forward_reroute(x, wr, b, wg, wu, wd, k, C)
    x64 = oracle.f64(x)
    want = np.zeros_like(out)
    moved = 0
    for t in range(T):
        for j in range(k):
            q = t * k + j
            e = int(rr.expert[q])
            if e < 0:
                continue
            moved += int(rr.round[q] > 0)
            _, y = oracle.expert_ffn(x64[t][None, :], wg[e], wu[e], wd[e])
            want[t] += w[t, j] * y[0]
            if not np.array_equal(xp[dest[q]], x64[t]):
                return False
    return bool(moved > 0 and np.allclose(out, want, rtol=1e-11, atol=1e-13))


def pin_expert_choice_map_argsort(seed=22, T=23, E=5, C=6):
    """The [T, E] row map built independently: expert e keeps the first C tokens of a stable
    descending argsort of its fp32 scores (library routine), listed in ascending token id; the
    i-th of them sits at row e*C + i; every other entry is -1."""
    rng = np.random.default_rng(seed)
    logits = rng.normal(size=(T, E))
    ec = oracle.expert_choice(logits, C)
    S = torch.softmax(torch.from_numpy(logits), dim=1).numpy().astype(np.float32)
    want = np.full((T, E), -1, dtype=np.int64)
    for e in range(E):
        picks = np.sort(np.argsort(-S[:, e], kind="stable")[:C])
        want[picks, e] = e * C + np.arange(C)
    got = oracle.expert_choice_map(ec, T)
    return bool(got.shape == (T, E) and np.array_equal(got, want))


def pin_ec_margin_enforcement(seed=23, T=300, E=6, C=40, gap=5e-4):
    """After enforce_ec_margin, every expert's C-th and (C+1)-th largest scores (library softmax over
    the experts, library descending sort) are at least `gap` (relative) apart, and the inputs needed
    redraws to get there."""
    w = syn.Workload("ecm", T=T, d=64, E=E, k=1, F=64)
    x, wr, b = syn.router_inputs(w, seed)

    def worst(xx):
        l = torch.nn.functional.linear(xx.double(), wr.double(), b.double() if b is not None else None)
        srt = torch.sort(torch.softmax(l, dim=1), dim=0, descending=True).values
        return float(((srt[C - 1] - srt[C]) / srt[C - 1]).min())
    before = worst(x)
    n = oracle.enforce_ec_margin(x, wr, b, C, lambda t, a: syn.x_row_redraw(w, seed, t, a), min_rel_gap=gap)
    return bool(before < gap and n > 0 and worst(x) >= gap)


def pin_silu_library():
    z = np.linspace(-30, 30, 2001)
    ref = torch.nn.functional.silu(torch.from_numpy(z)).numpy()
    return bool(np.allclose(oracle.silu(z), ref, rtol=1e-14, atol=1e-300) and oracle.silu(np.zeros(1))[0] == 0)


def pin_dispatch_invariants(seed=7, capacity=0):
    T, E, k = 50, 5, 2
    ids = syn.lognormal_topk_ids(E, T, k, 1.0, seed=seed).numpy()
    counts = oracle.histogram(ids, E)
    segs = oracle.plain_segments(counts, capacity)
    dest, src = oracle.dispatch_positions(ids, segs, E)
    flat = ids.ravel()
    kept = dest >= 0
    rows = int(segs.offsets[-1])
    ok = sorted(dest[kept].tolist()) == list(range(rows))
    ok &= all(src[dest[q]] == q for q in np.nonzero(kept)[0])
    off = segs.offsets
    for e in range(E):
        seg_src = src[off[e]:off[e + 1]]
        ok &= bool((flat[seg_src] == e).all()) and bool((np.diff(seg_src) > 0).all())
        want = min(counts[e], capacity) if capacity else counts[e]
        ok &= (off[e + 1] - off[e]) == want
    if capacity:
        ok &= int((~kept).sum()) == int(np.maximum(counts - capacity, 0).sum())
    else:
        ok &= bool(kept.all())
    return bool(ok)


def _plan_check(ids, E, R, S, k, B):
    counts = oracle.histogram(ids, E)
    segs, stats = oracle.balanced_plan(counts, R, S, k, B)
    dest, src = oracle.dispatch_positions(ids, segs, E)
    flat = ids.ravel()
    CAP = S * k
    n_per_group = E // R + B
    off = segs.offsets
    ok = bool((dest >= 0).all()) and sorted(dest.tolist()) == list(range(R * CAP))
    for g in range(R):
        ok &= int(off[(g + 1) * n_per_group] - off[g * n_per_group]) == CAP
    for s, e in enumerate(segs.expert):
        rows = src[off[s]:off[s + 1]]
        if e < 0:
            ok &= len(rows) == 0
        else:
            ok &= bool((flat[rows] == e).all())
    epg = E // R
    seg_group = np.repeat(np.arange(R), n_per_group)
    row_group = np.empty(R * CAP, dtype=np.int64)
    for s in range(len(segs.expert)):
        row_group[off[s]:off[s + 1]] = seg_group[s]
    moved = int((row_group[dest] != flat // epg).sum())
    loads = np.array([counts[g * epg:(g + 1) * epg].sum() for g in range(R)])
    lower_bound = int(np.maximum(loads - CAP, 0).sum())
    ok &= moved == lower_bound == stats.migrated_rows
    return ok, stats, loads


def pin_plan_moonep_table(sigmas=(0.5, 1.0, 2.0, 5.0)):
    """E=256, R=8, S=2048, k=8 (the MoonEP page's experiment): every group gets exactly S*k."""
    E, R, S, k, B = 256, 8, 2048, 8, 32
    for sigma in sigmas:
        ids = syn.lognormal_topk_ids(E, R * S, k, sigma, seed=11).numpy()
        ok, stats, loads = _plan_check(ids, E, R, S, k, B)
        if not ok:
            return False
    return True


def pin_plan_uniform():
    """Perfectly even routing needs no migration and no replica (sigma = 0 row)."""
    E, R, S, k, B = 256, 8, 2048, 8, 32
    ids = syn.uniform_roundrobin_ids(E, R * S, k).numpy()
    ok, stats, loads = _plan_check(ids, E, R, S, k, B)
    return ok and stats.migrated_rows == 0 and stats.replicas_used == 0 and (loads == S * k).all()


def pin_plan_toy_skew():
    """8 experts on 4 groups, top-1, 100 tokens, 70 on group 0's two experts, 10 on each other group.

    Busiest group: 70 tokens = 7x the others and 2.8x the mean of 25; the
    plan gives every group 25 rows and moves 45 of 100 rows.
    """
    ids = np.array([0] * 35 + [1] * 35 + [2] * 5 + [3] * 5 + [4] * 5 + [5] * 5 + [6] * 5 + [7] * 5)
    ids = ids.reshape(100, 1)
    ok, stats, loads = _plan_check(ids, E=8, R=4, S=25, k=1, B=4)
    ok &= list(loads) == [70, 10, 10, 10] and loads.max() / loads.mean() == 2.8
    ok &= loads.max() == 7 * loads[1:].max() and stats.migrated_rows == 45
    return bool(ok)


# --------------------------------------------------------------------------- the tests

def test_worked_top2_example():
    assert pin_worked_example()


def test_topk_brute_force():
    assert pin_topk_brute_force()


def test_topk_ties_go_to_lower_id():
    logits = np.array([[1.0, 3.0, 3.0, 2.0, 3.0]])
    assert list(oracle.topk_ids(logits, 3)[0]) == [1, 2, 4]


def test_topk_fp32_decision():
    # 1e-9 apart in fp64 but equal in fp32: the decision is taken in fp32, so the lower id wins
    logits = np.array([[1.0, 1.0 + 1e-9]])
    assert list(oracle.topk_ids(logits, 1)[0]) == [0]


def test_weights_equal_full_softmax_then_renorm():
    assert pin_weights_full_softmax()


def test_weights_softmax_all_variant():
    assert pin_weights_softmax_all()


def test_k1_weight_is_one():
    logits = np.random.default_rng(0).normal(size=(20, 8))
    w = oracle.topk_weights(logits, oracle.topk_ids(logits, 1))
    assert (w == 1.0).all()


def test_router_logits_match_library_linear():
    assert pin_router_logits_library()


def test_histogram():
    assert pin_histogram_bincount()


def test_rank_is_stable_sort_position():
    assert pin_rank_stable_sort()


def test_dispatch_invariants_no_capacity():
    assert pin_dispatch_invariants(capacity=0)


def test_dispatch_invariants_capacity():
    assert pin_dispatch_invariants(capacity=14)


def test_capacity_closed_form_skewed():
    w = syn.SKEWED
    assert oracle.capacity_rows(w.capacity_factor, w.T, w.k, w.E) == 320
    assert oracle.capacity_rows(0.0, 10, 2, 4) == 0
    assert oracle.capacity_rows(1.0, 10, 2, 4) == 5
    assert oracle.capacity_rows(1.0, 10, 2, 3) == 7


def test_silu():
    assert pin_silu_library()


def test_expert_choice_brute_force():
    assert pin_expert_choice_brute_force()


def test_expert_choice_layer_equals_loop():
    assert pin_expert_choice_layer_eager()


def test_expert_choice_capacity_above_tokens():
    logits = np.random.default_rng(3).normal(size=(5, 3))
    ec = oracle.expert_choice(logits, 99)
    assert all(list(p) == [0, 1, 2, 3, 4] for p in ec.picks)


def test_reroute_worked_example():
    assert pin_reroute_worked_example()


def test_reroute_without_overflow_is_top_k():
    assert pin_reroute_without_overflow()


def test_reroute_invariants():
    assert pin_reroute_invariants()


def test_reroute_positions_worked_example():
    assert pin_reroute_positions_worked()


def test_reroute_layer_equals_eager_pair_loop():
    assert pin_layer_reroute_eager()


def test_expert_choice_map_from_argsort():
    assert pin_expert_choice_map_argsort()


def test_expert_choice_margin_enforcement():
    assert pin_ec_margin_enforcement()


def test_shared_expert_adds_a_dense_ffn():
    assert pin_shared_expert_additive()


def test_layer_equals_eager_loop():
    assert pin_layer_equals_eager(capacity=0)


def test_layer_equals_eager_loop_with_capacity():
    assert pin_layer_equals_eager(capacity=5)


def test_dense_ffn_e1_k1():
    assert pin_dense_ffn_e1k1()


def test_plan_moonep_experiment_invariants():
    assert pin_plan_moonep_table()


def test_plan_uniform_routing_moves_nothing():
    assert pin_plan_uniform()


def test_plan_toy_skew_example():
    assert pin_plan_toy_skew()


def test_plan_infeasible_raises():
    ids = np.array([0] * 70 + [2] * 10 + [4] * 10 + [6] * 10).reshape(100, 1)
    with pytest.raises(oracle.PlanInfeasible):
        oracle.balanced_plan(oracle.histogram(ids, 8), 4, 25, 1, 0)


def test_plan_segment_count():
    assert oracle.num_segments(256, 8, 32) == 512
    assert oracle.num_segments(64, 0, 0) == 64


def test_margin_enforcement():
    w = syn.Workload("m", T=400, d=64, E=16, k=4, F=64)
    x, wr, b = syn.router_inputs(w, 3)
    before = oracle.margin_violations(oracle.router_logits(x, wr, b), w.k, 1e-3).sum()
    n = oracle.enforce_margin(x, wr, b, w.k, lambda t, a: syn.x_row_redraw(w, 3, t, a))
    after = oracle.margin_violations(oracle.router_logits(x, wr, b), w.k, 1e-3).sum()
    assert n == before and after == 0


# --------------------------------------------------------------------------- planted mistakes

def _mut_silu_sign(z):
    return z / (1.0 + np.exp(z))


def _mut_weights_no_renorm(logits64, ids):
    p = np.exp(logits64 - logits64.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    return np.take_along_axis(p, ids, axis=1)


def _mut_topk_ascending(logits64, k):
    return np.argsort(np.asarray(logits64).astype(np.float32), axis=1, kind="stable")[:, :k]


def _mut_histogram_offby1(ids, E):
    c = np.bincount(np.asarray(ids).ravel(), minlength=E)
    c[0] += 1
    return c


def _mut_rank_unstable(ids, E):
    flat = np.asarray(ids).ravel()
    rank = np.empty(flat.size, dtype=np.int64)
    seen = np.zeros(E, dtype=np.int64)
    for q in range(flat.size - 1, -1, -1):
        rank[q] = seen[flat[q]]
        seen[flat[q]] += 1
    return rank


_orig_expert_ffn = om.expert_ffn


def _mut_down_transposed(x_rows64, w_gate_e, w_up_e, w_down_e):
    wg, wu, wd = om.f64(w_gate_e), om.f64(w_up_e), om.f64(w_down_e)
    h = om.silu(x_rows64 @ wg.T) * (x_rows64 @ wu.T)
    return h, h @ wd   # wrong: W_down used untransposed


def _mut_logits_no_bias(x, w_router, bias=None):
    return om.f64(x) @ om.f64(w_router).T


_orig_combine = om.combine
_orig_weights = om.topk_weights


def _mut_combine_unweighted(yp64, dest, weights64, T, k):
    return _orig_combine(yp64, dest, np.ones_like(weights64), T, k)

def _mut_shared_transposed(x, w_gate_s, w_up_s, w_down_s):
    return om.expert_ffn(om.f64(x), w_up_s, w_gate_s, w_down_s)[1]   # gate and up swapped


_orig_candidate_order = om.candidate_order


def _mut_candidates_ascending(logits32_row):
    return _orig_candidate_order(-np.asarray(logits32_row))   # worst candidate first


_orig_reroute = om.reroute_overflow


def _mut_reroute_keeps_full(ids, logits64, C):
    rr = _orig_reroute(ids, logits64, C)
    rr.assigned = np.minimum(rr.assigned + 1, C + 1)   # one row too many somewhere
    return rr


_orig_expert_choice = om.expert_choice


def _mut_ec_keeps_weakest(logits64, capacity):
    return _orig_expert_choice(-np.asarray(logits64, dtype=np.float64), capacity)   # picks the lowest scores


_orig_reroute_positions = om.reroute_positions


def _mut_reroute_positions_next_offset(rr):
    segs, dest, src = _orig_reroute_positions(rr)
    off = segs.offsets
    dest = np.where(rr.expert >= 0, off[np.maximum(rr.expert, 0) + 1] + rr.slot, -1)   # off[e+1] for off[e]
    return segs, dest, src


_orig_layer_reroute = om.layer_forward_reroute


def _mut_layer_reroute_drops_moved(x, w_router, bias, w_gate, w_up, w_down, k, capacity):
    r = list(_orig_layer_reroute(x, w_router, bias, w_gate, w_up, w_down, k, capacity))
    rr, dest = r[3], r[5]
    dest = np.where(rr.round > 0, -1, dest)          # moved pairs treated as dropped
    r[10] = om.combine(r[9], dest, r[2], r[0].shape[0], k)
    return tuple(r)


_orig_ec_map = om.expert_choice_map


def _mut_ec_map_left_boundary(ec, T):
    E = len(ec.picks)
    m = np.full((T, E), -1, dtype=np.int64)
    for r in range(len(ec.src)):
        e = int(np.searchsorted(ec.segs.offsets, r, side="left") - 1)   # first row of a segment -> previous expert
        m[ec.src[r], e] = r
    return m


MUTATIONS = [
    ("silu", _mut_silu_sign, [pin_silu_library, pin_dense_ffn_e1k1]),
    ("topk_weights", _mut_weights_no_renorm, [pin_worked_example, pin_weights_full_softmax]),
    ("topk_ids", _mut_topk_ascending, [pin_worked_example, pin_topk_brute_force]),
    ("histogram", _mut_histogram_offby1, [pin_histogram_bincount]),
    ("expert_rank", _mut_rank_unstable, [pin_rank_stable_sort, pin_dispatch_invariants]),
    ("expert_ffn", _mut_down_transposed, [pin_dense_ffn_e1k1]),
    ("router_logits", _mut_logits_no_bias, [pin_router_logits_library]),
    ("combine", _mut_combine_unweighted, [pin_layer_equals_eager]),
    ("shared_expert", _mut_shared_transposed, [pin_shared_expert_additive]),
    ("topk_weights_softmax_all", lambda l, i: _orig_weights(l, i), [pin_weights_softmax_all]),
    ("expert_scores", lambda l: np.exp(l) / np.exp(l).sum(0, keepdims=True),   # softmax over tokens
     [pin_expert_choice_brute_force, pin_expert_choice_layer_eager]),
    ("expert_choice", _mut_ec_keeps_weakest, [pin_expert_choice_brute_force, pin_expert_choice_layer_eager]),
    ("candidate_order", _mut_candidates_ascending, [pin_reroute_worked_example, pin_reroute_invariants]),
    ("reroute_overflow", _mut_reroute_keeps_full, [pin_reroute_worked_example, pin_reroute_invariants]),
    ("reroute_positions", _mut_reroute_positions_next_offset, [pin_reroute_positions_worked, pin_layer_reroute_eager]),
    ("layer_forward_reroute", _mut_layer_reroute_drops_moved, [pin_layer_reroute_eager]),
    ("expert_choice_map", _mut_ec_map_left_boundary, [pin_expert_choice_map_argsort]),
    ("ec_margin_violations", lambda S, capacity, min_rel_gap: np.zeros(np.asarray(S).shape[1], dtype=bool),
     [pin_ec_margin_enforcement]),   # never asks for a redraw
]


@pytest.mark.parametrize("name,mutant,pins", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistakes_are_caught(monkeypatch, name, mutant, pins):
    monkeypatch.setattr(om, name, mutant)
    monkeypatch.setattr(oracle, name, mutant)
    results = []
    for pin in pins:
        try:
            results.append(pin())
        except Exception:
            results.append(False)
    assert not all(results), f"planted mistake in {name} went unnoticed"


# --------------------------------------------------------------------------- randomised sweeps

def test_plan_invariants_random_shapes():
    """The plan's invariants over random group counts, group sizes, replica budgets and skews:
    exact S*k rows per group, every pair placed once in a segment of its expert, the minimum
    number of migrated rows; an infeasible budget raises, and the same counts with B = E (room
    for any piece list) plan."""
    rng = np.random.default_rng(123)
    planned = infeasible = 0
    for _ in range(60):
        R = int(rng.integers(1, 7))
        E = R * int(rng.integers(1, 6))
        k = int(rng.integers(1, min(E, 4) + 1))
        S = int(rng.integers(1, 40))
        B = int(rng.integers(0, 4))
        sigma = float(rng.choice([0.0, 0.5, 1.5, 4.0]))
        ids = syn.lognormal_topk_ids(E, R * S, k, sigma, seed=int(rng.integers(1 << 30))).numpy()
        try:
            ok, _, _ = _plan_check(ids, E, R, S, k, B)
            assert ok
            planned += 1
        except oracle.PlanInfeasible:
            infeasible += 1
            ok, _, _ = _plan_check(ids, E, R, S, k, E)
            assert ok
    assert planned > 10 and infeasible > 0


def test_dispatch_invariants_random_shapes():
    """Stable counting-sort placement over random shapes and capacities: dest is a bijection onto
    the kept rows, each segment holds its expert's first min(count, C) pairs in q order (the
    positions of numpy's stable argsort), and dropped pairs are exactly the excess."""
    rng = np.random.default_rng(321)
    for _ in range(80):
        E = int(rng.integers(1, 40))
        k = int(rng.integers(1, min(E, 8) + 1))
        T = int(rng.integers(1, 300))
        ids = syn.lognormal_topk_ids(E, T, k, float(rng.choice([0.0, 1.0, 3.0])),
                                     seed=int(rng.integers(1 << 30))).numpy()
        counts = oracle.histogram(ids, E)
        C = int(rng.integers(0, 2 * T * k // E + 2))
        segs = oracle.plain_segments(counts, C)
        dest, src = oracle.dispatch_positions(ids, segs, E)
        flat = ids.ravel()
        order = np.argsort(flat, kind="stable")           # q order inside each expert
        starts = np.concatenate([[0], np.cumsum(counts)])
        off = segs.offsets
        for e in range(E):
            qs = order[starts[e]:starts[e + 1]]
            keep = len(qs) if C == 0 else min(len(qs), C)
            assert (dest[qs[:keep]] == off[e] + np.arange(keep)).all()
            assert (dest[qs[keep:]] == -1).all()
            assert (src[off[e]:off[e + 1]] == qs[:keep]).all()
        assert int((dest < 0).sum()) == (0 if C == 0 else int(np.maximum(counts - C, 0).sum()))
