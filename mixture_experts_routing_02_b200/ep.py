"""Expert parallelism across R ranks: the host-side plumbing around the moe_ep_* calls.

The balanced plan's R groups are R ranks (one GPU each): rank g owns the experts homed in
group g plus B replica weight slots and computes exactly S*k rows.  Every step of the layer
runs in the library's kernels; this module only moves the small things between ranks with
torch.distributed (the [E] counts of every rank, once the buffers' peer addresses) and
orders the steps with stream-ordered collectives:

    route + histogram  ->  counts all-gather  ->  moe_ep_plan  ->  moe_ep_prefetch_weights
    ->  moe_ep_dispatch (rows stored into their owners' final slots)  ->  barrier
    ->  moe_ep_expert_ffn  ->  barrier  ->  moe_ep_combine (output rows read from the owners)

("가장 바쁜 랭크가 속도를 정합니다: MoonEP의 계획 코드를 직접 돌려봤습니다", sections "이 기술은
무엇인가" and "설치 및 통합"; "5.3 Expert Parallelism", section "2. 디스패처 엔지니어링": the
counts are exchanged first, then the tokens.)

* ``gather_counts`` / ``gather_addresses``: the exchanges, on any process group (gloo on CPU
  tensors, NCCL on CUDA tensors).
* ``VirtualRanks``: R ranks on ONE GPU.  Every rank has its own buffers; the dispatch and the
  combine of all ranks run as one launch each (the kernels never wait for another rank), the
  way an R-GPU group runs them rank by rank.
* ``EpRank``: one rank of an R-GPU group, its receive buffers and weight slots in
  symmetric memory (torch.distributed._symmetric_memory) so that every rank has the others'
  addresses; the barriers are NCCL all-reduces on the compute stream.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import mixture_experts_routing_02_b200 as moe

__all__ = ["gather_counts", "gather_addresses", "ep_shape", "VirtualRanks", "EpRank"]


def gather_counts(counts_local, group=None):
    """counts_all [R, E]: row r = rank r's [E] expert counts, the same table on every rank."""
    import torch
    import torch.distributed as dist
    R = dist.get_world_size(group)
    parts = [torch.empty_like(counts_local) for _ in range(R)]
    dist.all_gather(parts, counts_local.contiguous(), group=group)
    return torch.stack(parts)


def gather_addresses(address: int, group=None) -> List[int]:
    """Every rank's value of `address` (a device address of a peer-mapped buffer), in rank order."""
    import torch
    import torch.distributed as dist
    R = dist.get_world_size(group)
    dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    mine = torch.tensor([int(address)], dtype=torch.int64, device=dev)
    parts = [torch.empty_like(mine) for _ in range(R)]
    dist.all_gather(parts, mine, group=group)
    return [int(p.item()) for p in parts]


def ep_shape(R: int, S: int, d: int, E: int, k: int, F: int, B: int, route_flags: int = 0,
             out_dtype: int = moe.DTYPE_F32):
    """The shape of the moe_ep_* calls: T = R*S tokens over R ranks (groups), B replica slots."""
    return moe.shape(R * S, d, E, k, F, n_groups=R, replica_slots=B, route_flags=route_flags, out_dtype=out_dtype)


def _rank_shape(s):
    """The single-rank shape of the routing calls: S tokens, no plan."""
    R = s.n_groups
    return moe.shape(s.T // R, s.d_model, s.n_experts, s.top_k, s.d_ff, route_flags=s.route_flags,
                     out_dtype=s.out_dtype)


class _RankBuffers:
    """Device buffers of one rank."""

    def __init__(self, s, device, allocate=None):
        import torch
        R, E, k, d, F, B = s.n_groups, s.n_experts, s.top_k, s.d_model, s.d_ff, s.replica_slots
        S = s.T // R
        n_loc = E // R + B
        alloc = allocate or (lambda shape, dtype: torch.empty(shape, dtype=dtype, device=device))
        i32 = lambda n: torch.zeros(n, dtype=torch.int32, device=device)
        self.ids = i32((S, k))
        self.w = torch.zeros(S, k, dtype=torch.float32, device=device)
        self.dest = i32(S * k)
        self.seg_expert, self.seg_slot, self.seg_offsets = i32(n_loc), i32(n_loc), i32(n_loc + 1)
        self.hp = torch.empty(S * k, F, dtype=torch.bfloat16, device=device)
        # buffers other ranks write into or read from: receive rows, their pair index, expert outputs
        self.xp = alloc((S * k, d), torch.bfloat16)
        self.src = alloc((S * k,), torch.int32)
        self.yp = alloc((S * k, d), torch.float32)
        self.out = torch.empty(S, d, dtype=torch.bfloat16 if s.out_dtype == moe.DTYPE_BF16 else torch.float32,
                               device=device)
        route_ws = moe.moe_route_workspace_size(_rank_shape(s))
        self.route_ws = torch.empty(route_ws, dtype=torch.uint8, device=device) if route_ws else None


def _weight_slots(s, r, wg, wu, wd, device, allocate=None):
    """Rank r's weight slots [E/R + B, ...] with its home experts in the first E/R slots."""
    import torch
    R, E, B = s.n_groups, s.n_experts, s.replica_slots
    epg = E // R
    out = []
    for w in (wg, wu, wd):
        shape = (epg + B,) + tuple(w.shape[1:])
        t = allocate(shape, torch.bfloat16) if allocate else torch.empty(shape, dtype=torch.bfloat16, device=device)
        t[:epg].copy_(w[r * epg:(r + 1) * epg])
        if B:
            t[epg:].zero_()
        out.append(t)
    return out


class VirtualRanks:
    """R expert-parallel ranks on one GPU (see the module docstring).

    wg, wu: [E, F, d], wd: [E, d, F] -- all experts' weights; rank r's slots start with its home
    experts.  forward(x_ranks, w_router, bias) takes the R ranks' [S, d] inputs and returns their
    [S, d] outputs.
    """

    def __init__(self, s, wg, wu, wd, device="cuda"):
        import torch
        self.s = s
        self.R = s.n_groups
        self.rs = _rank_shape(s)
        self.dev = torch.device(device)
        self.bufs = [_RankBuffers(s, self.dev) for _ in range(self.R)]
        slots = [_weight_slots(s, r, wg, wu, wd, self.dev) for r in range(self.R)]
        self.wg, self.wu, self.wd = ([sl[m] for sl in slots] for m in range(3))
        self.counts_all = torch.zeros(self.R, s.n_experts, dtype=torch.int32, device=self.dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.dev)

    def forward(self, x_ranks: Sequence, w_router, bias=None, stream=None, mark=None):
        """mark(name), if given, is called after each phase is enqueued (e.g. to record an event)."""
        s, b = self.s, self.bufs
        mark = mark or (lambda name: None)
        for r in range(self.R):
            moe.moe_route_ws(self.rs, x_ranks[r], w_router, bias, None, b[r].ids, b[r].w, self.status, b[r].route_ws,
                             stream)
            moe.moe_histogram(self.rs, b[r].ids, self.counts_all[r], stream)   # the counts "all-gather"
        mark("route")
        for r in range(self.R):
            moe.moe_ep_plan(s, r, self.counts_all, None, b[r].seg_expert, b[r].seg_slot, b[r].seg_offsets,
                            self.status, stream)
        mark("plan")
        for r in range(self.R):
            moe.moe_ep_prefetch_weights(s, r, b[r].seg_expert, b[r].seg_offsets, self.wg, self.wu, self.wd, stream)
        mark("prefetch")
        moe.moe_ep_dispatch(s, 0, list(x_ranks), [x.ids for x in b], self.counts_all, [x.dest for x in b],
                            [x.xp for x in b], [x.src for x in b], self.status, stream)
        mark("dispatch")
        for r in range(self.R):
            moe.moe_ep_expert_ffn(s, b[r].xp, b[r].seg_slot, b[r].seg_offsets, self.wg[r], self.wu[r], self.wd[r],
                                  b[r].hp, b[r].yp, self.status, stream)
        mark("ffn")
        moe.moe_ep_combine(s, 0, [x.yp for x in b], [x.dest for x in b], [x.w for x in b], [x.out for x in b],
                           stream)
        mark("combine")
        return [x.out for x in b]

    def kernel_launches(self) -> int:
        """Kernels one forward launches (route GEMM + routing, histogram, plan, prefetch per rank; one
        dispatch; gate/up + down per rank; one combine)."""
        route = 2 if self.bufs[0].route_ws is not None else 1
        return self.R * (route + 1 + 1 + 1 + 2) + 2


class EpRank:
    """One rank of an expert-parallel group of R processes, one GPU each.

    The buffers that other ranks write (Xp, src) or read (Yp, the home weight slots) live in
    symmetric memory; their peer addresses come from the rendezvous.  wg, wu, wd: this rank's
    home experts' weights ([E/R, F, d], [E/R, F, d], [E/R, d, F]).
    """

    def __init__(self, s, wg_home, wu_home, wd_home, group=None):
        import torch
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
        self.s, self.group = s, group
        self.R = s.n_groups
        self.rank = dist.get_rank(group)
        if dist.get_world_size(group) != self.R:
            raise ValueError("the shape's n_groups must equal the group's size")
        self.rs = _rank_shape(s)
        self.dev = torch.device("cuda", torch.cuda.current_device())
        handles = []

        def symmetric(shape, dtype):
            t = symm_mem.empty(*shape, dtype=dtype, device=self.dev)
            handles.append(symm_mem.rendezvous(t, group if group is not None else dist.group.WORLD))
            return t

        self.b = _RankBuffers(s, self.dev, allocate=symmetric)
        self.wg, self.wu, self.wd = _weight_slots_home(s, wg_home, wu_home, wd_home, symmetric)
        self.peers = [list(h.buffer_ptrs) for h in handles]   # xp, src, yp, wg, wu, wd: R addresses each
        self.counts = torch.zeros(s.n_experts, dtype=torch.int32, device=self.dev)
        self.counts_all = torch.zeros(self.R, s.n_experts, dtype=torch.int32, device=self.dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.dev)
        self._flag = torch.zeros(1, dtype=torch.int32, device=self.dev)

    def _barrier(self):
        # stream-ordered on NCCL.  Two per step suffice: the next step's counts all-gather completes
        # only once every rank has finished this step's combine, so the next dispatch (which writes
        # the peers' Xp / src) and expert GEMMs (which write Yp) cannot overtake a peer's reads.
        import torch.distributed as dist
        dist.all_reduce(self._flag, group=self.group)

    def forward(self, x, w_router, bias=None):
        import torch.distributed as dist
        s, b, lib = self.s, self.b, moe.load_library()
        moe.moe_route_ws(self.rs, x, w_router, bias, None, b.ids, b.w, self.status, b.route_ws)
        moe.moe_histogram(self.rs, b.ids, self.counts)
        dist.all_gather_into_tensor(self.counts_all, self.counts, group=self.group)
        moe.moe_ep_plan(s, self.rank, self.counts_all, None, b.seg_expert, b.seg_slot, b.seg_offsets, self.status)
        xp, src, yp, wg, wu, wd = (_addr_table(p) for p in self.peers)
        moe._check("moe_ep_prefetch_weights", lib.moe_ep_prefetch_weights(
            moe.ctypes.byref(s), self.rank, moe._ptr(b.seg_expert), moe._ptr(b.seg_offsets), wg, wu, wd,
            moe._stream(None)))
        moe._check("moe_ep_dispatch", lib.moe_ep_dispatch(
            moe.ctypes.byref(s), self.rank, 1, moe._ptr_table([x]), moe._ptr_table([b.ids]),
            moe._ptr(self.counts_all), moe._ptr_table([b.dest]), xp, src, moe._ptr(self.status), moe._stream(None)))
        self._barrier()                       # every rank's rows have arrived
        moe.moe_ep_expert_ffn(s, b.xp, b.seg_slot, b.seg_offsets, self.wg, self.wu, self.wd, b.hp, b.yp, self.status)
        self._barrier()                       # every owner's Yp is complete
        moe._check("moe_ep_combine", lib.moe_ep_combine(
            moe.ctypes.byref(s), self.rank, 1, yp, moe._ptr_table([b.dest]), moe._ptr_table([b.w]),
            moe._ptr_table([b.out]), moe._stream(None)))
        return b.out


def _weight_slots_home(s, wg_home, wu_home, wd_home, allocate):
    R, E, B = s.n_groups, s.n_experts, s.replica_slots
    epg = E // R
    out = []
    for w in (wg_home, wu_home, wd_home):
        t = allocate((epg + B,) + tuple(w.shape[1:]), w.dtype)
        t[:epg].copy_(w)
        if B:
            t[epg:].zero_()
        out.append(t)
    return out


def _addr_table(addresses: Sequence[int]):
    return (moe.ctypes.c_void_p * len(addresses))(*addresses)
