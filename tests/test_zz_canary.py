"""Out-of-range writes.  Every buffer a call writes is placed inside a larger allocation whose
bytes on both sides (4 KB each) and whose unused interior rows hold a canary byte; after the
call those bytes must be unchanged.  The calls run one by one as moe_layer_fwd makes them (route,
dispatch, gate/up, down, combine, and the expert-choice and re-routing variants), and their
output must equal moe_layer_fwd's bit for bit (the same kernels on the same inputs, none of
which depends on timing).

compute-sanitizer is not available on these GPUs, so this is the check for stray stores.
The file sorts last so that it runs after the parity tests.
"""
import numpy as np
import pytest
import torch

import mixture_experts_routing_02_b200 as moe
from mixture_experts_routing_02_b200 import synthetic as syn

from gpu_cases import dev, make_case, moe_shape, run_layer, to_np

pytestmark = pytest.mark.gpu

PAD = 4096          # canary bytes before and after each buffer (keeps the buffer 256-byte aligned)
CANARY = 0xA5


class Guarded:
    """A tensor of `shape` and `dtype` inside canary bytes."""

    def __init__(self, shape, dtype):
        shape = tuple(int(s) for s in shape)
        n = int(np.prod(shape))
        assert n > 0
        self.nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((PAD + self.nbytes + PAD,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.raw[PAD:PAD + self.nbytes].view(dtype).view(*shape)

    def check(self, what, unused_from=None):
        """The bytes around the buffer (and, with unused_from, the interior bytes from that offset
        on, e.g. rows past the used ones) still hold the canary."""
        raw = self.raw.cpu().numpy()
        head, tail = raw[:PAD], raw[PAD + self.nbytes:]
        assert (head == CANARY).all(), f"{what}: {int((head != CANARY).sum())} bytes written before the buffer"
        assert (tail == CANARY).all(), f"{what}: {int((tail != CANARY).sum())} bytes written after the buffer"
        if unused_from is not None:
            rest = raw[PAD + unused_from:PAD + self.nbytes]
            assert (rest == CANARY).all(), f"{what}: {int((rest != CANARY).sum())} bytes written in unused rows"


def _guard_all(bufs, skip=()):
    return {k: Guarded(*v) for k, v in bufs.items() if k not in skip}


def _run_topk(case, s):
    """Route, dispatch, gate/up, down and combine call by call; returns the guards and the rows used."""
    w = case.w
    T, d, E, k, F = w.T, w.d, w.E, w.k, w.F
    n_seg, rows = moe.moe_layout(s)
    rr = bool(s.route_flags & moe.ROUTE_REROUTE)
    route_ws_bytes = moe.moe_route_workspace_size(s)
    disp_bytes = moe.moe_workspace_size(s)[0]
    g = _guard_all(dict(
        ids=((T, k), torch.int32), wts=((T, k), torch.float32), counts=((E,), torch.int32),
        seg_e=((n_seg,), torch.int32), seg_o=((n_seg + 1,), torch.int32), seg_f=((n_seg,), torch.int32),
        dest=((T * k,), torch.int32), src=((rows,), torch.int32), xp=((rows, d), torch.bfloat16),
        hp=((rows, F), torch.bfloat16), yp=((rows, d), torch.float32),
        out=((T, d), torch.bfloat16 if s.out_dtype == moe.DTYPE_BF16 else torch.float32),
        logits=((T, E), torch.float32), route_ws=((max(route_ws_bytes, 1),), torch.uint8),
        dws=((max(disp_bytes, 1),), torch.uint8)))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x, w_r, bias = dev(case.x), dev(case.w_r), dev(case.bias)
    wg, wu, wd = dev(case.wg), dev(case.wu), dev(case.wd)
    moe.moe_route_ws(s, x, w_r, bias, g["logits"].t if rr else None, g["ids"].t, g["wts"].t, status,
                     g["route_ws"].t if route_ws_bytes else None)
    if rr:
        moe.moe_dispatch_reroute(s, x, g["ids"].t, g["logits"].t, g["counts"].t, g["seg_e"].t, g["seg_o"].t,
                                 g["seg_f"].t, g["dest"].t, g["src"].t, g["xp"].t, status, g["dws"].t)
    else:
        moe.moe_dispatch(s, x, g["ids"].t, 0, g["counts"].t, g["seg_e"].t, g["seg_o"].t, g["seg_f"].t,
                         g["dest"].t, g["src"].t, g["xp"].t, status, g["dws"].t)
    moe.moe_expert_gate_up(s, g["xp"].t, g["seg_e"].t, g["seg_o"].t, wg, wu, g["hp"].t, status)
    moe.moe_expert_down(s, g["hp"].t, g["seg_e"].t, g["seg_o"].t, wd, g["yp"].t, status)
    moe.moe_combine(s, g["yp"].t, g["dest"].t, g["wts"].t, g["out"].t)
    torch.cuda.synchronize()
    assert status.item() == 0
    used = int(g["seg_o"].t[-1].item())
    return g, used, rr


CASES = [
    # count dispatch with a capacity that drops pairs
    syn.Workload("capacity", T=500, d=128, E=16, k=2, F=192, zipf_s=1.2, capacity_factor=1.0),
    # count dispatch with the balanced plan (replica segments)
    syn.Workload("plan", T=512, d=128, E=16, k=4, F=128, zipf_s=1.2, n_groups=4, replica_slots=8),
    # more than 65536 pairs: the look-back dispatch
    syn.Workload("lookback", T=9000, d=64, E=64, k=8, F=64, zipf_s=0.5),
    # long segments: several row tiles per expert
    syn.Workload("pairs", T=700, d=192, E=3, k=2, F=320, zipf_s=1.0),
    # overflow re-routing
    syn.Workload("reroute", T=600, d=128, E=8, k=2, F=128, zipf_s=1.2, capacity_factor=1.0, reroute=True),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_topk_calls_write_only_their_buffers(cuda_ok, w):
    case = make_case(w, seed=31)
    s = moe_shape(w)
    g, used, rr = _run_topk(case, s)
    d, F = w.d, w.F
    for name, guard in g.items():
        unused = None
        if name == "xp":
            unused = used * d * 2
        elif name == "hp":
            unused = used * F * 2
        elif name == "yp":
            unused = used * d * 4
        guard.check(name, unused)
    ref = run_layer(case)
    assert ref["status"] == 0
    assert np.array_equal(to_np(g["out"].t), to_np(ref["out"])), "call-by-call output differs from moe_layer_fwd"


def test_bf16_output_writes_only_its_buffer(cuda_ok):
    """With out_dtype = bf16 the combine writes T * d * 2 bytes and nothing around them."""
    w = CASES[0]
    case = make_case(w, seed=33)
    s = moe_shape(w)
    s.out_dtype = moe.DTYPE_BF16
    g, used, rr = _run_topk(case, s)
    assert g["out"].t.dtype == torch.bfloat16
    g["out"].check("out")
    ref = run_layer(case, out_dtype=moe.DTYPE_BF16)
    assert ref["status"] == 0
    assert torch.equal(g["out"].t, ref["out"]), "call-by-call output differs from moe_layer_fwd"


def test_expert_choice_calls_write_only_their_buffers(cuda_ok):
    w = syn.Workload("ec", T=700, d=128, E=8, k=2, F=192, zipf_s=1.0, capacity_factor=1.0, expert_choice=True)
    case = make_case(w, seed=32)
    s = moe_shape(w)
    T, d, E, F = w.T, w.d, w.E, w.F
    n_seg, rows = moe.moe_layout(s)
    route_ws_bytes = moe.moe_route_workspace_size(s)
    g = _guard_all(dict(
        scores=((E, T), torch.float32), seg_e=((n_seg,), torch.int32), seg_o=((n_seg + 1,), torch.int32),
        src=((rows,), torch.int32), row_w=((rows,), torch.float32), emap=((T, E), torch.int32),
        xp=((rows, d), torch.bfloat16), hp=((rows, F), torch.bfloat16), yp=((rows, d), torch.float32),
        out=((T, d), torch.float32), route_ws=((max(route_ws_bytes, 1),), torch.uint8)))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x, w_r, bias = dev(case.x), dev(case.w_r), dev(case.bias)
    moe.moe_route_scores_ws(s, x, w_r, bias, g["scores"].t, status, g["route_ws"].t if route_ws_bytes else None)
    moe.moe_expert_choose(s, g["scores"].t, x, g["seg_e"].t, g["seg_o"].t, g["src"].t, g["row_w"].t, g["emap"].t,
                          g["xp"].t)
    moe.moe_expert_gate_up(s, g["xp"].t, g["seg_e"].t, g["seg_o"].t, dev(case.wg), dev(case.wu), g["hp"].t, status)
    moe.moe_expert_down(s, g["hp"].t, g["seg_e"].t, g["seg_o"].t, dev(case.wd), g["yp"].t, status)
    moe.moe_combine_expert_choice(s, g["yp"].t, g["emap"].t, g["row_w"].t, None, g["out"].t)
    torch.cuda.synchronize()
    assert status.item() == 0
    for name, guard in g.items():
        guard.check(name)
    ref = run_layer(case)
    assert ref["status"] == 0
    assert np.array_equal(to_np(g["out"].t), to_np(ref["out"])), "call-by-call output differs from moe_layer_fwd"
