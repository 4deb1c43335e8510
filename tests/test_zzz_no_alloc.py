"""moe_dispatch_static: the dispatch for callers that cannot allocate device memory
(for example code running during CUDA-graph stream capture, where cudaMalloc is
not allowed, or a runtime plug-in that is handed only its input and output
buffers).  It takes its look-back scratch from a static array inside the
library instead of a caller-provided workspace.

The array is read by every dispatch path that needs scratch: the single-launch
look-back dispatch (more than 65536 pairs, no plan), a dispatch on given plan
tables (plan_ready = 1), a balanced plan of up to 16 groups (per-group counts,
then the grouped dispatch), and a balanced plan of more than 16 groups and more
than 2^20 pairs (histogram partials, plan, look-back ranks, row copies).  Each case first runs a call of a
different shape so that stale ticket and look-back words are left in the array,
then calls moe_dispatch_static twice in a row; both results must equal
moe_dispatch's (with its own workspace) and the oracle's bit for bit.

This file sorts last, so a run that stops at the first failure has run every
other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn


def _buffers(s, T, k, d, E):
    n_seg, rows = moe.moe_layout(s)
    mk = lambda n: torch.full((max(n, 1),), -7, dtype=torch.int32, device="cuda")
    return dict(counts=mk(E), seg_expert=mk(n_seg), seg_offsets=mk(n_seg + 1), seg_first_rank=mk(n_seg),
                dest=mk(T * k), src=mk(rows),
                xp=torch.full((rows, d), float("nan"), dtype=torch.bfloat16, device="cuda"),
                status=torch.zeros(1, dtype=torch.int32, device="cuda"))


def _i32(a):
    return torch.from_numpy(np.asarray(a, dtype=np.int32)).cuda()


def _run(fn, s, x, ids, b, plan_ready, **kw):
    fn(s, x, ids, plan_ready, b["counts"], b["seg_expert"], b["seg_offsets"], b["seg_first_rank"], b["dest"],
       b["src"], b["xp"], b["status"], **kw)


CASES = [
    # no plan, more than 65536 pairs: the single-launch look-back dispatch (ticket + per-tile words)
    dict(name="lookback", T=9000, d=64, E=64, k=8, R=0, B=0, C=0, sigma=0.5, plan_ready=0),
    # the same with a capacity that drops pairs
    dict(name="lookback-capacity", T=9000, d=64, E=32, k=8, R=0, B=0, C=2000, sigma=1.2, plan_ready=0),
    # tables given by the caller: look-back ranks and row copies after clearing the words
    dict(name="plan-given", T=800, d=128, E=32, k=4, R=4, B=8, C=0, sigma=2.0, plan_ready=1),
    # a balanced plan of up to 16 groups: per-group counts in the array, then the grouped dispatch
    dict(name="plan-groups", T=1200, d=192, E=32, k=4, R=4, B=8, C=0, sigma=2.0, plan_ready=0),
    # more than 16 groups and more than 2^20 pairs: histogram partials, plan, look-back ranks, copies
    dict(name="large-plan", T=140032, d=64, E=32, k=8, R=32, B=4, C=0, sigma=1.0, plan_ready=0),
    # at most 65536 pairs and no plan: the count dispatch, which needs no scratch at all
    dict(name="count", T=999, d=128, E=16, k=2, R=0, B=0, C=90, sigma=1.0, plan_ready=0),
]


def _oracle(c, ids_np):
    counts = oracle.histogram(ids_np, c["E"])
    if c["R"]:
        segs, _ = oracle.balanced_plan(counts, c["R"], c["T"] // c["R"], c["k"], c["B"])
    else:
        segs = oracle.plain_segments(counts, c["C"])
    dest, src = oracle.dispatch_positions(ids_np, segs, c["E"])
    return counts, segs, dest, src


@pytest.mark.gpu
@pytest.mark.parametrize("c", CASES, ids=[c["name"] for c in CASES])
def test_static_scratch_dispatch(cuda_ok, c):
    T, d, E, k = c["T"], c["d"], c["E"], c["k"]
    s = moe.shape(T, d, E, k, 64, capacity=c["C"], n_groups=c["R"], replica_slots=c["B"])
    ids = syn.lognormal_topk_ids(E, T, k, c["sigma"], seed=21).cuda()
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(22)).to(torch.bfloat16).cuda()
    ids_np = ids.view(T, k).cpu().numpy()
    counts, segs, dest, src = _oracle(c, ids_np)
    used = int(segs.offsets[-1])

    # leave stale words of another shape in the array: a look-back dispatch of other sizes
    s_dirty = moe.shape(9500, 64, 40, 8, 64, capacity=1500)   # 76000 pairs: the look-back path
    ids_dirty = syn.lognormal_topk_ids(40, 9500, 8, 3.0, seed=23).cuda()
    dirty = _buffers(s_dirty, 9500, 8, 64, 40)
    _run(moe.moe_dispatch_static, s_dirty, torch.ones(9500, 64, dtype=torch.bfloat16, device="cuda"), ids_dirty,
         dirty, 0)

    def given(b):
        if c["plan_ready"]:
            b["counts"].copy_(_i32(counts))
            b["seg_expert"].copy_(_i32(segs.expert))
            b["seg_offsets"].copy_(_i32(segs.offsets))
            b["seg_first_rank"].copy_(_i32(segs.first_rank))
        return b

    ref = given(_buffers(s, T, k, d, E))
    ws = torch.empty(moe.moe_workspace_size(s)[0], dtype=torch.uint8, device="cuda")
    _run(moe.moe_dispatch, s, x, ids, ref, c["plan_ready"], ws=ws)
    torch.cuda.synchronize()
    assert ref["status"].item() == 0 and dirty["status"].item() == 0

    want = dict(counts=counts, seg_expert=segs.expert, seg_offsets=segs.offsets, seg_first_rank=segs.first_rank,
                dest=dest)
    xp_want = x[torch.from_numpy(src // k).cuda()]
    for call in range(2):
        got = given(_buffers(s, T, k, d, E))
        _run(moe.moe_dispatch_static, s, x, ids, got, c["plan_ready"])
        torch.cuda.synchronize()
        assert got["status"].item() == 0, f"call {call}"
        for name, w in want.items():
            assert torch.equal(got[name], ref[name]), f"call {call}: {name} differs from moe_dispatch"
            assert (got[name].cpu().numpy() == w).all(), f"call {call}: {name} differs from the oracle"
        assert torch.equal(got["src"][:used], ref["src"][:used]), f"call {call}: src differs from moe_dispatch"
        assert (got["src"][:used].cpu().numpy() == src).all(), f"call {call}: src differs from the oracle"
        assert torch.equal(got["xp"][:used], ref["xp"][:used]), f"call {call}: rows differ from moe_dispatch"
        assert torch.equal(got["xp"][:used], xp_want), f"call {call}: rows differ from the oracle's permutation"


def test_static_scratch_rejects_oversized_shapes():
    """Shapes whose look-back scratch exceeds the 4 MiB array fail before anything is enqueued."""
    lib = moe.load_library()
    s = moe.shape(1 << 20, 64, 256, 1, 64)        # 4096 tiles x 256 experts x 4 B > 4 MiB
    fake = ctypes.c_void_p(1 << 20)               # never dereferenced: the size check comes first
    rc = lib.moe_dispatch_static(ctypes.byref(s), fake, fake, 0, fake, fake, fake, fake, fake, fake, fake,
                                 None, None)
    assert rc == 2 and moe.moe_status_string(rc).startswith("MOE_ERR_UNSUPPORTED")
