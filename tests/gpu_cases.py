"""Helpers of the GPU parity tests: seeded inputs (with the top-k margin rule),
device buffers, the tolerance of floating-point outputs, and the oracle side
of each comparison.  Imported only by tests."""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

# Floating-point outputs (bf16 in, fp32 accumulate) against the fp64 oracle:
# max-abs error <= 2e-2 * RMS(reference) and mean relative error (sum|err| / sum|ref|) <= 5e-3.
MAX_ABS_OF_RMS = 2e-2
MEAN_REL = 5e-3


def check_close(got, ref, what="", max_abs_of_rms=MAX_ABS_OF_RMS, mean_rel=MEAN_REL):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    if ref.size == 0:
        return
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    denom = float(np.abs(ref).sum())
    max_abs = float(err.max())
    rel = float(err.sum()) / denom if denom > 0 else float(err.sum())
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert max_abs <= max_abs_of_rms * max(rms, 1e-30), f"{what}: max-abs {max_abs:.3e} > {max_abs_of_rms} * rms {rms:.3e}"
    assert rel <= mean_rel, f"{what}: mean-rel {rel:.3e} > {mean_rel}"


def check_bf16_storage(got, ref, what=""):
    """An intermediate stored in bf16 (Hp): one round-to-nearest to bf16 of an fp32 value that
    differs from the fp64 reference by fp32 accumulation error.  Bound per element:
    2^-7 |ref| (one bf16 ulp: half an ulp for the rounding, and the fp32 value may sit across a
    rounding boundary from the fp64 one) + 2^-12 RMS(ref) for the accumulation error of values
    near zero (about 30x the typical sqrt(K) * 2^-24 accumulation error at K <= 16384)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    if ref.size == 0:
        return
    rms = float(np.sqrt(np.mean(ref * ref)))
    bound = 2.0 ** -7 * np.abs(ref) + 2.0 ** -12 * rms
    bad = np.abs(got - ref) > bound
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond one bf16 rounding, worst " \
                          f"{float((np.abs(got - ref) / np.maximum(bound, 1e-300)).max()):.3f}x the bound"


def check_layer_output(got, ref, dest, T, k, what="out"):
    """Layer output against the oracle.  Rows of tokens whose k pairs were all dropped (capacity)
    must be exactly 0; the tolerance of check_close applies to the other rows, whose RMS is the
    scale of the computed values (a tensor of mostly structural zeros would otherwise shrink it)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    dropped = (np.asarray(dest).reshape(T, k) < 0).all(axis=1)
    assert (got[dropped] == 0).all(), f"{what}: rows of fully dropped tokens are not zero"
    check_close(got[~dropped], ref[~dropped], what)


def check_yp_elementwise(got, ref_result, case, what="Yp"):
    """Yp, an intermediate the pages do not bound, against the bound its arithmetic gives: its
    operand Hp is rounded to bf16 once, so per element |err| <= 2^-7 * (|h| . |W_d[e]|^T) (one
    bf16 ulp carried through the contraction; it covers the fp32 accumulation too), plus a tiny
    absolute term; and mean-rel <= 5e-3.  Unlike max-abs <= 2e-2 * RMS it does not tighten as
    the number of elements (and so the reach of the largest error) grows."""
    got = np.asarray(got, dtype=np.float64)
    r = ref_result
    used = int(r.segs.offsets[-1])
    ref = r.yp[:used]
    a = np.zeros_like(ref)
    off = r.segs.offsets
    for s, e in enumerate(r.segs.expert):
        if e >= 0 and off[s + 1] > off[s]:
            a[off[s]:off[s + 1]] = np.abs(r.hp[off[s]:off[s + 1]]) @ np.abs(oracle.f64(case.wd[int(e)])).T
    err = np.abs(got[:used] - ref)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    bad = err > 2.0 ** -7 * a + 1e-7 * max(rms, 1e-30)
    assert np.isfinite(got[:used]).all(), f"{what}: non-finite values"
    assert not bad.any(), f"{what}: {int(bad.sum())} elements above the bound"
    denom = float(np.abs(ref).sum())
    if denom > 0:
        assert float(err.sum()) / denom <= MEAN_REL, f"{what}: mean-rel {float(err.sum()) / denom:.3e}"


def check_output_elementwise(got, ref_result, case, what="out"):
    """Per-element bound on the layer output, derived from its one bf16 rounding (Hp, the operand of
    the down projection):  |got - ref| <= 2^-7 * sum_j |w_j| * (|h_j| . |W_d[e_j]|^T)  (+ a tiny
    absolute term), with 2^-7 = one bf16 ulp covering the rounding and the fp32 accumulation; plus
    the mean relative error <= 5e-3.  Unlike max-abs <= 2e-2 * RMS it does not depend on how
    heavy-tailed the output is (deep capacity drops with unrenormalised weights)."""
    got = np.asarray(got, dtype=np.float64)
    r = ref_result
    rows, d = r.hp.shape[0], r.out.shape[1]
    a = np.zeros((rows, d))
    off = r.segs.offsets
    for s, e in enumerate(r.segs.expert):
        if e >= 0 and off[s + 1] > off[s]:
            a[off[s]:off[s + 1]] = np.abs(r.hp[off[s]:off[s + 1]]) @ np.abs(oracle.f64(case.wd[int(e)])).T
    T, k = r.out.shape[0], r.ids.shape[1]
    bound = 2.0 ** -7 * oracle.combine(a, r.dest, np.abs(r.weights), T, k)
    rms = float(np.sqrt(np.mean(r.out ** 2))) if r.out.size else 0.0
    err = np.abs(got - r.out)
    bad = err > bound + 1e-7 * max(rms, 1e-30)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert not bad.any(), f"{what}: {int(bad.sum())} elements above the bound (worst {float((err / (bound + 1e-30)).max()):.2f}x)"
    denom = float(np.abs(r.out).sum())
    if denom > 0:
        assert float(err.sum()) / denom <= MEAN_REL, f"{what}: mean-rel {float(err.sum()) / denom:.3e}"


def capacity_rows(w: syn.Workload) -> int:
    return oracle.capacity_rows(w.capacity_factor, w.T, w.k, w.E)


def moe_shape(w: syn.Workload, capacity: Optional[int] = None):
    C = capacity_rows(w) if capacity is None else capacity
    flags = (moe.ROUTE_EXPERT_CHOICE if w.expert_choice else 0) | (moe.ROUTE_REROUTE if w.reroute else 0)
    return moe.shape(w.T, w.d, w.E, w.k, w.F, capacity=C, n_groups=w.n_groups, replica_slots=w.replica_slots,
                     route_flags=flags)


@dataclasses.dataclass
class Case:
    w: syn.Workload
    x: torch.Tensor        # CPU bf16, margin-enforced
    w_r: torch.Tensor      # CPU bf16
    bias: Optional[torch.Tensor]
    wg: torch.Tensor       # bf16 on `weights_device`
    wu: torch.Tensor
    wd: torch.Tensor


def make_case(w: syn.Workload, seed: int = 0, weights_device="cpu", margin=True) -> Case:
    x, w_r, bias = syn.router_inputs(w, seed)
    if margin and w.E > 1:
        redraw = lambda t, a: syn.x_row_redraw(w, seed, t, a)
        if w.expert_choice:
            oracle.enforce_ec_margin(x, w_r, bias, capacity_rows(w), redraw)
        elif w.reroute:
            # re-routed pairs go down each token's whole logit order: keep all of it 1e-3 apart
            oracle.enforce_margin(x, w_r, bias, w.E - 1, redraw)
        else:
            oracle.enforce_margin(x, w_r, bias, w.k, redraw)
    wg, wu, wd = syn.expert_weights(w, seed, device=weights_device)
    return Case(w, x, w_r, bias, wg, wu, wd)


def dev(t, device="cuda"):
    return None if t is None else t.to(device).contiguous()


def i32(n, device="cuda"):
    return torch.zeros(max(int(n), 1), dtype=torch.int32, device=device)


def to_np(t):
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def run_layer(case: Case, capacity=None, stream=None, route_flags=0, out_dtype=moe.DTYPE_F32):
    """moe_layer_fwd through the C ABI; returns the output (fp32 or bf16 on the device) and every
    intermediate (CPU)."""
    w = case.w
    s = moe_shape(w, capacity)
    s.route_flags |= route_flags
    s.out_dtype = out_dtype
    n_seg, rows = moe.moe_layout(s)
    _, layer_bytes = moe.moe_workspace_size(s)
    ws = torch.empty(layer_bytes, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((w.T, w.d), float("nan"), device="cuda",
                     dtype=torch.bfloat16 if out_dtype == moe.DTYPE_BF16 else torch.float32)
    x, w_r, bias = dev(case.x), dev(case.w_r), dev(case.bias)
    wg, wu, wd = dev(case.wg), dev(case.wu), dev(case.wd)
    moe.moe_layer_fwd(s, x, w_r, bias, wg, wu, wd, out, status, ws, stream=stream)
    torch.cuda.synchronize()
    v = moe.moe_layer_views(s, ws)

    def view(addr, n, dtype, shape=None):
        base = ws.data_ptr()
        off = addr - base
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        t = ws[off:off + nbytes].view(dtype)
        return t.view(*shape) if shape else t

    T, k = w.T, w.k
    common = dict(
        out=out, status=int(status.item()), n_seg=n_seg, rows=rows, ws=ws, x_dev=x,
        seg_expert=view(v.seg_expert, n_seg, torch.int32).cpu(),
        seg_offsets=view(v.seg_offsets, n_seg + 1, torch.int32).cpu(),
        src=view(v.src, rows, torch.int32).cpu(),
        xp=view(v.xp, rows * w.d, torch.bfloat16, (rows, w.d)),
        hp=view(v.hp, rows * w.F, torch.bfloat16, (rows, w.F)),
        yp=view(v.yp, rows * w.d, torch.float32, (rows, w.d)),
    )
    if s.route_flags & moe.ROUTE_EXPERT_CHOICE:
        return dict(common,
                    scores=view(v.scores, w.E * T, torch.float32, (w.E, T)).cpu(),
                    emap=view(v.emap, T * w.E, torch.int32, (T, w.E)).cpu(),
                    row_w=view(v.row_w, rows, torch.float32).cpu())
    res = dict(
        out=out, status=int(status.item()), n_seg=n_seg, rows=rows, ws=ws, x_dev=x,
        ids=view(v.topk_ids, T * k, torch.int32, (T, k)).cpu(),
        w=view(v.topk_w, T * k, torch.float32, (T, k)).cpu(),
        counts=view(v.counts, w.E, torch.int32).cpu(),
        seg_expert=view(v.seg_expert, n_seg, torch.int32).cpu(),
        seg_offsets=view(v.seg_offsets, n_seg + 1, torch.int32).cpu(),
        seg_first_rank=view(v.seg_first_rank, n_seg, torch.int32).cpu(),
        dest=view(v.dest, T * k, torch.int32).cpu(),
        src=view(v.src, rows, torch.int32).cpu(),
        xp=view(v.xp, rows * w.d, torch.bfloat16, (rows, w.d)),
        hp=view(v.hp, rows * w.F, torch.bfloat16, (rows, w.F)),
        yp=view(v.yp, rows * w.d, torch.float32, (rows, w.d)),
    )
    return res


def oracle_segments(case: Case, counts, capacity=None):
    w = case.w
    if w.n_groups:
        segs, _ = oracle.balanced_plan(counts, w.n_groups, w.T // w.n_groups, w.k, w.replica_slots)
    else:
        segs = oracle.plain_segments(counts, capacity_rows(w) if capacity is None else capacity)
    return segs


def expert_rows(pairs, wg, wu, wd, with_bound=False):
    """{key: (h, y)} -- or (h, y, |h| . |W_d[e]|^T) with with_bound -- for (key, x_row64, expert)
    pairs, evaluated in fp64 one expert's weights at a time."""
    by_e = {}
    for key, xrow, e in pairs:
        by_e.setdefault(int(e), []).append((key, xrow))
    out = {}
    for e, items in by_e.items():
        g64, u64, d64 = (oracle.f64(t[e].cpu()) for t in (wg, wu, wd))
        xs = np.stack([x for _, x in items])
        h = oracle.silu(xs @ g64.T) * (xs @ u64.T)
        y = h @ d64.T
        a = np.abs(h) @ np.abs(d64).T if with_bound else None
        for i, (key, _) in enumerate(items):
            out[key] = (h[i], y[i], a[i]) if with_bound else (h[i], y[i])
    return out
