"""Expert parallelism across R ranks, run as R virtual ranks on one GPU (each rank with its
own buffers; the dispatch and the combine of all ranks as one launch each, the kernels never
waiting for another rank).

Against the oracle's balanced plan over the R*S tokens in rank order (group g = rank g):
the plan's tables of every rank, dest, src and the received rows bit for bit; the replica
weight slots bit for bit against their home experts; Hp, Yp and the output within tolerance.
Against the single-GPU balanced-plan layer: the same rows in the same slots and the same
expert outputs, bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import ep
from mixture_experts_routing_02_b200 import synthetic as syn

from gpu_cases import check_bf16_storage, check_close, check_layer_output, make_case, run_layer, to_np

pytestmark = pytest.mark.gpu

CASES = [
    syn.Workload("ep-r4", T=4 * 300, d=128, E=32, k=4, F=128, zipf_s=1.2, n_groups=4, replica_slots=8),
    syn.Workload("ep-r2-ragged", T=2 * 513, d=192, E=8, k=2, F=192, zipf_s=1.5, n_groups=2, replica_slots=3),
    syn.Workload("ep-r8", T=8 * 96, d=64, E=64, k=8, F=64, zipf_s=1.2, n_groups=8, replica_slots=8),
    syn.Workload("ep-r16-uniform", T=16 * 40, d=64, E=16, k=2, F=64, n_groups=16, replica_slots=2),
]


def _run(case, out_dtype=moe.DTYPE_F32):
    w = case.w
    R, S = w.n_groups, w.tokens_per_group
    s = ep.ep_shape(R, S, w.d, w.E, w.k, w.F, w.replica_slots, out_dtype=out_dtype)
    vr = ep.VirtualRanks(s, case.wg.cuda(), case.wu.cuda(), case.wd.cuda())
    x = case.x.cuda()
    bias = case.bias.cuda() if case.bias is not None else None
    outs = vr.forward([x[r * S:(r + 1) * S] for r in range(R)], case.w_r.cuda(), bias)
    torch.cuda.synchronize()
    return s, vr, outs


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_virtual_ranks_match_the_oracle(cuda_ok, w):
    case = make_case(w, seed=3)
    ref = oracle.layer_forward(case.x, case.w_r, case.bias, case.wg, case.wu, case.wd, w.k,
                               n_groups=w.n_groups, replica_slots=w.replica_slots)
    s, vr, outs = _run(case)
    assert vr.status.item() == 0
    R, S, k, E, B = w.n_groups, w.tokens_per_group, w.k, w.E, w.replica_slots
    cap, epg = S * k, E // R
    pg = epg + B
    for r, b in enumerate(vr.bufs):
        rows = slice(r * cap, (r + 1) * cap)
        assert (b.ids.cpu().numpy() == ref.ids[r * S:(r + 1) * S]).all(), f"rank {r}: top-k ids"
        assert (vr.counts_all[r].cpu().numpy() == oracle.histogram(ref.ids[r * S:(r + 1) * S], E)).all()
        segs_e = ref.segs.expert[r * pg:(r + 1) * pg]
        segs_o = ref.segs.offsets[r * pg:(r + 1) * pg + 1] - r * cap
        assert (b.seg_expert.cpu().numpy() == segs_e).all(), f"rank {r}: seg_expert"
        assert (b.seg_offsets.cpu().numpy() == segs_o).all(), f"rank {r}: seg_offsets"
        live = (segs_e >= 0) & (np.diff(segs_o) > 0)
        assert (b.seg_slot.cpu().numpy() == np.where(live, np.arange(pg), -1)).all(), f"rank {r}: seg_slot"
        assert (b.dest.cpu().numpy() == ref.dest[r * S * k:(r + 1) * S * k]).all(), f"rank {r}: dest"
        assert (b.src.cpu().numpy() == ref.src[rows]).all(), f"rank {r}: src"
        assert (to_np(b.xp) == ref.xp[rows]).all(), f"rank {r}: received rows"
        # replica slots hold exact copies of their experts' weights
        for j in range(B):
            e = int(segs_e[epg + j])
            if e >= 0 and segs_o[epg + j + 1] > segs_o[epg + j]:
                for mine, full in ((vr.wg[r], case.wg), (vr.wu[r], case.wu), (vr.wd[r], case.wd)):
                    assert torch.equal(mine[epg + j].cpu(), full[e]), f"rank {r}: replica slot {j} (expert {e})"
        check_bf16_storage(to_np(b.hp), ref.hp[rows], f"rank {r}: Hp")
        check_close(to_np(b.yp), ref.yp[rows], f"rank {r}: Yp")
        check_layer_output(to_np(outs[r]), ref.out[r * S:(r + 1) * S], ref.dest[r * S * k:(r + 1) * S * k], S, k,
                           f"rank {r}: out")


@pytest.mark.parametrize("w", CASES[:2], ids=[w.name for w in CASES[:2]])
def test_virtual_ranks_equal_the_single_gpu_plan(cuda_ok, w):
    """R ranks reproduce the single-GPU balanced-plan layer: rank g's rows are rows [g*S*k, (g+1)*S*k)
    of the single-GPU Xp, and its expert outputs are the same bits."""
    case = make_case(w, seed=4)
    s, vr, _ = _run(case)
    one = run_layer(case)
    assert vr.status.item() == 0 and one["status"] == 0
    R, S, k = w.n_groups, w.tokens_per_group, w.k
    cap = S * k
    dest = np.concatenate([b.dest.cpu().numpy() for b in vr.bufs])
    assert (dest == one["dest"].numpy()).all()
    for r, b in enumerate(vr.bufs):
        rows = slice(r * cap, (r + 1) * cap)
        assert torch.equal(b.xp, one["xp"][rows]), f"rank {r}: rows differ from the single-GPU layout"
        assert torch.equal(b.yp, one["yp"][rows]), f"rank {r}: expert outputs differ from the single GPU's"


def test_virtual_ranks_bf16_output(cuda_ok):
    """out_dtype = bf16 through the expert-parallel combine: the fp32 combine rounded once."""
    w = CASES[0]
    case = make_case(w, seed=5)
    _, _, o32 = _run(case)
    _, _, o16 = _run(case, out_dtype=moe.DTYPE_BF16)
    for a, b in zip(o32, o16):
        assert b.dtype == torch.bfloat16 and torch.equal(b, a.to(torch.bfloat16))


def test_virtual_ranks_infeasible_plan(cuda_ok):
    """More replica pieces than slots: every rank reports MOE_DEV_ERR_PLAN, nothing is dispatched,
    the output is zero."""
    w = syn.Workload("ep-infeasible", T=4 * 64, d=64, E=16, k=2, F=64, zipf_s=3.0, n_groups=4, replica_slots=0)
    case = make_case(w, seed=6)
    with pytest.raises(oracle.PlanInfeasible):
        oracle.layer_forward(case.x, case.w_r, case.bias, case.wg, case.wu, case.wd, w.k, n_groups=4, replica_slots=0)
    _, vr, outs = _run(case)
    assert vr.status.item() & moe.DEV_ERR_PLAN
    for b, o in zip(vr.bufs, outs):
        assert (b.dest.cpu().numpy() == -1).all()
        assert (to_np(o) == 0).all()
