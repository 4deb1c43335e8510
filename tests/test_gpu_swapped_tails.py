"""The grouped expert GEMMs on segments whose last row tile is short.

In the down projection with d_ff <= 4096, a segment's last 128-row tile with at most 32 rows is
computed with the operands swapped (the weight tile as the 128-row operand, the tile's rows as the
narrow one).  These cases put every kind of tail next to each other -- 1, 15, 16, 17 rows
(swapped), 33, 64, 95, 96, 97, 127, 128 rows (not), whole tiles followed by a short tail, an empty
segment -- with output widths that end on a partial column tile and d_ff on both sides of 4096,
and compare Hp and Yp with the oracle's expert FFN ("5.3 Expert
Parallelism", section "3. 고도화된 최적화: 오버래핑(Overlapping) 및 GroupGEMM": one grouped GEMM
over every expert's rows)."""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

from gpu_cases import check_bf16_storage, check_yp_elementwise, dev, i32, make_case, moe_shape, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(cuda_ok):
    yield


# segment lengths (one segment per expert, in expert order); each list sums to T * k
SEGMENTS = {
    "short-tails": [1, 15, 16, 17, 33, 64, 95, 96, 97, 127, 128, 0, 150, 161, 224, 255, 268, 380, 297],
    "long-segments": [1000, 1025, 1119, 1120, 1152, 1151, 129, 96],
}


# d_ff = 4096 is the longest reduction that takes the swapped tails, 4160 the shortest that does not
@pytest.mark.parametrize("d,F", [(512, 384), (384, 320), (256, 128), (256, 4096), (256, 4160)])
@pytest.mark.parametrize("layout", sorted(SEGMENTS))
def test_expert_ffn_with_short_segment_tails(layout, d, F):
    lengths = SEGMENTS[layout]
    E, k = len(lengths), 2
    rows = int(sum(lengths))
    assert rows % k == 0
    w = syn.Workload("tails", T=rows // k, d=d, E=E, k=k, F=F)
    case = make_case(w, seed=11)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    expert = np.arange(E, dtype=np.int64)
    rng = np.random.default_rng(5)
    xp = torch.from_numpy(rng.standard_normal((rows, d)).astype(np.float32)).to(torch.bfloat16)
    xp64 = xp.float().numpy().astype(np.float64)
    segs = SimpleNamespace(offsets=offsets, expert=expert, length=np.diff(offsets))
    hp_ref, yp_ref = oracle.grouped_expert_ffn(xp64, segs, case.wg, case.wu, case.wd)

    s = moe_shape(w)
    n_seg, rows_alloc = moe.moe_layout(s)
    assert n_seg == E and rows_alloc >= rows
    hp = torch.empty(rows_alloc, F, dtype=torch.bfloat16, device="cuda")
    yp = torch.empty(rows_alloc, d, dtype=torch.float32, device="cuda")
    st = i32(1)
    moe.moe_expert_ffn(s, xp.cuda(), dev(torch.from_numpy(expert.astype(np.int32))),
                       dev(torch.from_numpy(offsets.astype(np.int32))), dev(case.wg), dev(case.wu), dev(case.wd),
                       hp, yp, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    check_bf16_storage(to_np(hp)[:rows], hp_ref, "Hp")
    ref = SimpleNamespace(segs=segs, hp=hp_ref, yp=yp_ref)
    check_yp_elementwise(to_np(yp), ref, case, "Yp")
