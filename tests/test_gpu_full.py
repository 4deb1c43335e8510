"""Full-size parity: the four large workloads at their real sizes, run through
moe_layer_fwd (the launch configuration the benchmark times).

Every index output (top-k ids, counts, segment tables, dest, src) is compared
with the oracle in full, bit for bit; every permuted row is checked to be an
exact copy of its token; floating-point outputs are compared on sampled rows
and tokens that the oracle evaluates one by one in fp64.  The layer output is
stored in the type the benchmark returns for the workload: bf16 where the bf16
output meets the stated tolerance (Workload.bf16_out), fp32 otherwise; the
balanced-plan layer's bf16 output is checked too and recorded as a measured miss.
"""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

from gpu_cases import (check_bf16_storage, check_close, check_layer_output, expert_rows, make_case, oracle_segments,
                       run_layer, to_np)

pytestmark = pytest.mark.gpu

FULL = [syn.MIXTRAL_LIKE, syn.DEEPSEEK_LIKE, syn.SKEWED, syn.BALANCED]


# (workload, output type): each workload in the type the benchmark returns it in, and the
# balanced-plan layer's bf16 output, which misses the tolerance (reported as an expected failure)
RUNS = [(w, moe.DTYPE_BF16 if w.bf16_out else moe.DTYPE_F32) for w in FULL] + [
    pytest.param(syn.BALANCED, moe.DTYPE_BF16, marks=pytest.mark.xfail(
        reason="measured miss of the stated tolerance: balanced-plan layer with a bf16 output, max-abs error "
               "2.04e-2 x RMS on the sampled tokens (rounding the output to bf16 adds up to half a bf16 ulp)",
        strict=False), id="balanced-plan-bf16")]


@pytest.mark.parametrize("w,out_dtype", RUNS,
                         ids=[f"{w.name}-{'bf16' if dt == moe.DTYPE_BF16 else 'f32'}" for w, dt in RUNS[:len(FULL)]]
                         + ["balanced-plan-bf16"])
def test_full_size_layer(cuda_ok, w, out_dtype):
    case = make_case(w, seed=0, weights_device="cuda")
    got = run_layer(case, out_dtype=out_dtype)
    want_dtype = torch.bfloat16 if out_dtype == moe.DTYPE_BF16 else torch.float32
    assert got["status"] == 0 and got["out"].dtype == want_dtype

    # routing of all T tokens
    logits, ids, wts = oracle.route(case.x, case.w_r, case.bias, w.k)
    assert (got["ids"].numpy() == ids).all(), "top-k ids differ"
    assert np.abs(got["w"].numpy() - wts).max() < 1e-4

    # dispatch tables and positions of all T*k pairs
    counts = oracle.histogram(ids, w.E)
    assert (got["counts"].numpy() == counts).all()
    segs = oracle_segments(case, counts)
    assert (got["seg_expert"].numpy() == segs.expert).all()
    assert (got["seg_offsets"].numpy() == segs.offsets).all()
    assert (got["seg_first_rank"].numpy() == segs.first_rank).all()
    dest, src = oracle.dispatch_positions(ids, segs, w.E)
    assert (got["dest"].numpy() == dest).all()
    used = int(segs.offsets[-1])
    assert (got["src"].numpy()[:used] == src).all()
    if w.n_groups:
        cap = w.tokens_per_group * w.k
        assert (np.diff(segs.offsets[:: w.E // w.n_groups + w.replica_slots]) == cap).all()

    # every dispatched row is an exact copy of its token's row (checked on the device)
    src_dev = torch.from_numpy(src.astype(np.int64)).cuda()
    assert torch.equal(got["xp"][:used], got["x_dev"][src_dev // w.k])

    # expert FFN on sampled rows: first, last and a middle row of a spread of segments
    rng = np.random.default_rng(0)
    live = [s for s in range(len(segs.expert)) if segs.length[s] > 0]
    pick = sorted(set(rng.choice(live, size=min(24, len(live)), replace=False).tolist()))
    rows = []
    for s in pick:
        a, b = int(segs.offsets[s]), int(segs.offsets[s + 1])
        rows += sorted({a, b - 1, (a + b) // 2})
    x64 = oracle.f64(case.x)
    row_expert = {r: int(segs.expert[np.searchsorted(segs.offsets, r, side="right") - 1]) for r in rows}
    ref_rows = expert_rows([(r, x64[src[r] // w.k], row_expert[r]) for r in rows], case.wg, case.wu, case.wd)
    rsel = torch.tensor(rows, device="cuda")
    check_bf16_storage(to_np(got["hp"][rsel]), np.stack([ref_rows[r][0] for r in rows]), "Hp (sampled rows)")
    check_close(to_np(got["yp"][rsel]), np.stack([ref_rows[r][1] for r in rows]), "Yp (sampled rows)")

    # layer output on sampled tokens, evaluated token by token (no dispatch)
    toks = sorted(set(rng.choice(w.T, size=12, replace=False).tolist()) | {0, w.T - 1})
    pairs = [((t, j), x64[t], ids[t, j]) for t in toks for j in range(w.k) if dest[t * w.k + j] >= 0]
    ref_pairs = expert_rows(pairs, case.wg, case.wu, case.wd)
    ref_out = np.zeros((len(toks), w.d))
    for i, t in enumerate(toks):
        for j in range(w.k):
            if (t, j) in ref_pairs:
                ref_out[i] += wts[t, j] * ref_pairs[(t, j)][1]
    sel_dest = np.concatenate([dest[t * w.k:(t + 1) * w.k] for t in toks])
    check_layer_output(to_np(got["out"][torch.tensor(toks, device="cuda")]), ref_out, sel_dest, len(toks), w.k,
                       "out (sampled tokens)")


def test_full_size_shared_expert(cuda_ok):
    """DeepSeek-like shape with one shared expert (F_s = 2048): sampled rows against the oracle."""
    w = syn.DEEPSEEK_LIKE
    Fs = 2048
    x, _, _ = syn.router_inputs(w, 0)
    gs, us, ds = syn.shared_expert_weights(w, Fs, 0)
    s = moe.shape(w.T, w.d, w.E, w.k, w.F)
    h_s = torch.empty(w.T, Fs, dtype=torch.bfloat16, device="cuda")
    y_s = torch.empty(w.T, w.d, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_shared_expert(s, Fs, x.cuda(), gs.cuda(), us.cuda(), ds.cuda(), h_s, y_s, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    rng = np.random.default_rng(1)
    toks = sorted(set(rng.choice(w.T, size=16, replace=False).tolist()) | {0, w.T - 1})
    ref = oracle.shared_expert(x[toks], gs, us, ds)
    check_close(to_np(y_s[torch.tensor(toks, device="cuda")]), ref, "shared expert (sampled tokens)")
