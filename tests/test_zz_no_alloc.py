"""moe_dispatch_static: the dispatch for callers that cannot allocate device memory
(for example code running during CUDA-graph stream capture, where cudaMalloc is
not allowed, or a runtime plug-in that is handed only its input and output
buffers).  It takes its look-back scratch from a static array inside the
library instead of a caller-provided workspace.  These tests call it through
the C ABI and require exactly the results of moe_dispatch, on two calls in a
row (the array keeps the previous call's contents, which each call must clear).
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn


def _buffers(s, T, k, d, E):
    n_seg, rows = moe.moe_layout(s)
    mk = lambda n: torch.full((max(n, 1),), -7, dtype=torch.int32, device="cuda")
    return dict(counts=mk(E), seg_expert=mk(n_seg), seg_offsets=mk(n_seg + 1), seg_first_rank=mk(n_seg),
                dest=mk(T * k), src=mk(rows),
                xp=torch.full((rows, d), float("nan"), dtype=torch.bfloat16, device="cuda"),
                status=torch.zeros(1, dtype=torch.int32, device="cuda"))


def _run(fn, s, x, ids, b, **kw):
    fn(s, x, ids, 0, b["counts"], b["seg_expert"], b["seg_offsets"], b["seg_first_rank"], b["dest"], b["src"],
       b["xp"], b["status"], **kw)


CASES = [
    # balanced plan over 4 groups with skewed routing; several look-back tiles and a ragged last one
    dict(T=1200, d=192, E=32, k=4, R=4, B=8, C=0, sigma=2.0),
    # plain layout with a capacity that drops pairs
    dict(T=999, d=128, E=16, k=2, R=0, B=0, C=90, sigma=1.0),
]


@pytest.mark.gpu
@pytest.mark.parametrize("c", CASES, ids=["plan", "capacity"])
def test_static_scratch_dispatch_equals_workspace_dispatch(cuda_ok, c):
    T, d, E, k = c["T"], c["d"], c["E"], c["k"]
    s = moe.shape(T, d, E, k, 64, capacity=c["C"], n_groups=c["R"], replica_slots=c["B"])
    ids = syn.lognormal_topk_ids(E, T, k, c["sigma"], seed=21).cuda()
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(22)).to(torch.bfloat16).cuda()

    ref = _buffers(s, T, k, d, E)
    ws = torch.empty(moe.moe_workspace_size(s)[0], dtype=torch.uint8, device="cuda")
    _run(moe.moe_dispatch, s, x, ids, ref, ws=ws)
    torch.cuda.synchronize()
    assert ref["status"].item() == 0
    used = int(ref["seg_offsets"][-1].item())

    for call in range(2):
        got = _buffers(s, T, k, d, E)
        _run(moe.moe_dispatch_static, s, x, ids, got)
        torch.cuda.synchronize()
        assert got["status"].item() == 0, f"call {call}"
        for name in ("counts", "seg_expert", "seg_offsets", "seg_first_rank", "dest"):
            assert torch.equal(got[name], ref[name]), f"call {call}: {name} differs"
        assert torch.equal(got["src"][:used], ref["src"][:used]), f"call {call}: src differs"
        assert torch.equal(got["xp"][:used], ref["xp"][:used]), f"call {call}: dispatched rows differ"


def test_static_scratch_rejects_oversized_shapes():
    """Shapes whose look-back scratch exceeds the 4 MiB array fail before anything is enqueued."""
    lib = moe.load_library()
    s = moe.shape(1 << 20, 64, 256, 1, 64)        # 4096 tiles x 256 experts x 4 B > 4 MiB
    fake = ctypes.c_void_p(1 << 20)               # never dereferenced: the size check comes first
    rc = lib.moe_dispatch_static(ctypes.byref(s), fake, fake, 0, fake, fake, fake, fake, fake, fake, fake,
                                 None, None)
    assert rc == 2 and moe.moe_status_string(rc).startswith("MOE_ERR_UNSUPPORTED")
