"""Python binding of the C ABI in ``include/moe_routing.h`` (libmoe_b200.so).

Argument marshalling only: every function takes torch CUDA tensors (or None
for a nullable pointer), passes their device addresses and the current CUDA
stream to the C call of the same name, and raises ``MoeError`` when the call
returns a status other than MOE_OK.  All computation happens in the library's
CUDA kernels; there is no fallback of any kind.  If the library has not been
built, the first call raises ``RuntimeError``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "MoeError", "MoeShape", "MoeLayerViews", "LIB_PATH", "SYMBOLS", "load_library", "shape",
    "moe_status_string", "moe_layout", "moe_workspace_size", "moe_route", "moe_route_from_logits",
    "moe_histogram", "moe_segments", "moe_plan_balanced", "moe_dispatch", "moe_dispatch_static", "moe_expert_gate_up",
    "moe_expert_down", "moe_expert_ffn", "moe_combine", "moe_combine_add", "moe_shared_expert", "moe_layer_fwd",
    "moe_route_scores", "moe_expert_choose", "moe_combine_expert_choice",
    "moe_route_workspace_size", "moe_route_ws", "moe_route_scores_ws", "moe_dispatch_reroute",
    "moe_layer_views", "moe_routing_stats", "STAT_NAMES", "MoeAux", "moe_layer_fwd_aux",
    "EP_MAX_RANKS", "moe_ep_sizes", "moe_ep_plan", "moe_ep_prefetch_weights", "moe_ep_dispatch", "moe_ep_expert_ffn",
    "moe_ep_combine",
    "DEV_ERR_PLAN", "DEV_ERR_TIMEOUT", "ROUTE_SOFTMAX_ALL", "ROUTE_EXPERT_CHOICE", "ROUTE_REROUTE",
    "DTYPE_F32", "DTYPE_BF16",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

DEV_ERR_PLAN = 0x1
DEV_ERR_TIMEOUT = 0x2


class MoeError(RuntimeError):
    pass


class MoeShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("T", "d_model", "n_experts", "top_k", "d_ff", "capacity", "n_groups", "replica_slots",
                 "route_flags", "out_dtype")]


class MoeAux(ctypes.Structure):
    """moe_aux_t: device addresses (or None) that moe_layer_fwd_aux copies the routing results to."""
    _fields_ = [(n, ctypes.c_void_p) for n in ("topk_ids", "topk_w", "counts", "seg_offsets", "dest", "stats")]


class MoeLayerViews(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("topk_ids", "topk_w", "counts", "seg_expert", "seg_offsets", "seg_first_rank", "dest",
                 "src", "xp", "hp", "yp", "dispatch_ws")] + [("dispatch_ws_bytes", ctypes.c_size_t)] + \
        [(n, ctypes.c_void_p) for n in ("scores", "emap", "row_w", "logits")]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_S = ctypes.POINTER(MoeShape)

# name -> argument types (return type is moe_status_t = int, except moe_status_string)
SYMBOLS = {
    "moe_status_string": [ctypes.c_int],
    "moe_layout": [_S, _P, _P],
    "moe_workspace_size": [_S, _P, _P],
    "moe_route": [_S, _P, _P, _P, _P, _P, _P, _P, _P],
    "moe_route_from_logits": [_S, _P, _P, _P, _P],
    "moe_histogram": [_S, _P, _P, _P],
    "moe_segments": [_S, _P, _P, _P, _P, _P],
    "moe_plan_balanced": [_S, _P, _P, _P, _P, _P, _P],
    "moe_dispatch": [_S, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "moe_dispatch_static": [_S, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "moe_testing_dispatch_stalled": [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "moe_expert_gate_up": [_S, _P, _P, _P, _P, _P, _P, _P, _P],
    "moe_testing_gemm_stalled": [_S, _P, _P, _P, _P, _P, _P, _P, _P],
    "moe_testing_reroute_stalled": [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "moe_expert_down": [_S, _P, _P, _P, _P, _P, _P, _P],
    "moe_expert_ffn": [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "moe_combine": [_S, _P, _P, _P, _P, _P],
    "moe_combine_add": [_S, _P, _P, _P, _P, _P, _P],
    "moe_shared_expert": [_S, _I, _P, _P, _P, _P, _P, _P, _P, _P],
    "moe_layer_fwd": [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "moe_layer_fwd_aux": [_S, _P, _P, _P, _P, _P, _P, _P, ctypes.POINTER(MoeAux), _P, _P, ctypes.c_size_t, _P],
    "moe_layer_views": [_S, _P, ctypes.POINTER(MoeLayerViews)],
    "moe_route_scores": [_S, _P, _P, _P, _P, _P, _P],
    "moe_expert_choose": [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "moe_combine_expert_choice": [_S, _P, _P, _P, _P, _P, _P],
    "moe_route_workspace_size": [_S, _P],
    "moe_route_ws": [_S, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "moe_route_scores_ws": [_S, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "moe_dispatch_reroute": [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "moe_routing_stats": [_S, _P, _P, _P, _P, _P],
    "moe_ep_sizes": [_S, _P, _P, _P],
    "moe_ep_plan": [_S, _I, _P, _P, _P, _P, _P, _P, _P],
    "moe_ep_prefetch_weights": [_S, _I, _P, _P, _P, _P, _P, _P],
    "moe_ep_dispatch": [_S, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P],
    "moe_ep_expert_ffn": [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "moe_ep_combine": [_S, _I, _I, _P, _P, _P, _P, _P],
}

# order of the values moe_routing_stats writes (MOE_STAT_* in the header)
STAT_NAMES = ("pairs", "rows", "dropped", "max_expert_load", "active_experts", "max_segment_rows",
              "max_group_load", "max_group_rows", "migrated_rows", "replicas_used")

_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoe_b200.so and declare every exported call (raises if it is missing)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run `python -m mixture_experts_routing_02_b200.build`")
    lib = ctypes.CDLL(path)
    for name, args in SYMBOLS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "moe_status_string" else ctypes.c_int
    if path == LIB_PATH:
        _lib = lib
    return lib


ROUTE_SOFTMAX_ALL = 0x1
ROUTE_EXPERT_CHOICE = 0x2
ROUTE_REROUTE = 0x4
DTYPE_F32 = 0
DTYPE_BF16 = 1


def shape(T, d_model, n_experts, top_k, d_ff, capacity=0, n_groups=0, replica_slots=0, route_flags=0,
          out_dtype=DTYPE_F32) -> MoeShape:
    """out_dtype: DTYPE_F32 or DTYPE_BF16, the element type of the layer output `out`."""
    return MoeShape(T, d_model, n_experts, top_k, d_ff, capacity, n_groups, replica_slots, route_flags, out_dtype)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor arguments must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(name: str, st: int):
    if st != 0:
        raise MoeError(f"{name}: {load_library().moe_status_string(st).decode()}")


def moe_status_string(st: int) -> str:
    return load_library().moe_status_string(st).decode()


def moe_layout(s: MoeShape):
    n_seg, rows = ctypes.c_int32(), ctypes.c_int32()
    _check("moe_layout", load_library().moe_layout(ctypes.byref(s), ctypes.byref(n_seg), ctypes.byref(rows)))
    return n_seg.value, rows.value


def moe_workspace_size(s: MoeShape):
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check("moe_workspace_size", load_library().moe_workspace_size(ctypes.byref(s), ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def moe_route(s, x, w_router, bias, logits, topk_ids, topk_w, status=None, stream=None):
    _check("moe_route", load_library().moe_route(
        ctypes.byref(s), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(logits), _ptr(topk_ids), _ptr(topk_w),
        _ptr(status), _stream(stream)))


def moe_route_from_logits(s, logits, topk_ids, topk_w, stream=None):
    _check("moe_route_from_logits", load_library().moe_route_from_logits(
        ctypes.byref(s), _ptr(logits), _ptr(topk_ids), _ptr(topk_w), _stream(stream)))


def moe_histogram(s, topk_ids, counts, stream=None):
    _check("moe_histogram", load_library().moe_histogram(ctypes.byref(s), _ptr(topk_ids), _ptr(counts),
                                                          _stream(stream)))


def moe_segments(s, counts, seg_expert, seg_offsets, seg_first_rank, stream=None):
    _check("moe_segments", load_library().moe_segments(
        ctypes.byref(s), _ptr(counts), _ptr(seg_expert), _ptr(seg_offsets), _ptr(seg_first_rank), _stream(stream)))


def moe_plan_balanced(s, counts, seg_expert, seg_offsets, seg_first_rank, status=None, stream=None):
    _check("moe_plan_balanced", load_library().moe_plan_balanced(
        ctypes.byref(s), _ptr(counts), _ptr(seg_expert), _ptr(seg_offsets), _ptr(seg_first_rank), _ptr(status),
        _stream(stream)))


def moe_dispatch(s, x, topk_ids, plan_ready, counts, seg_expert, seg_offsets, seg_first_rank, dest, src, xp,
                 status, ws, stream=None):
    _check("moe_dispatch", load_library().moe_dispatch(
        ctypes.byref(s), _ptr(x), _ptr(topk_ids), int(plan_ready), _ptr(counts), _ptr(seg_expert),
        _ptr(seg_offsets), _ptr(seg_first_rank), _ptr(dest), _ptr(src), _ptr(xp), _ptr(status), _ptr(ws),
        ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def moe_dispatch_static(s, x, topk_ids, plan_ready, counts, seg_expert, seg_offsets, seg_first_rank, dest, src, xp,
                        status, stream=None):
    """moe_dispatch with the library's own static scratch instead of a workspace (see the header)."""
    _check("moe_dispatch_static", load_library().moe_dispatch_static(
        ctypes.byref(s), _ptr(x), _ptr(topk_ids), int(plan_ready), _ptr(counts), _ptr(seg_expert),
        _ptr(seg_offsets), _ptr(seg_first_rank), _ptr(dest), _ptr(src), _ptr(xp), _ptr(status), _stream(stream)))


def moe_testing_dispatch_stalled(s, x, topk_ids, counts, seg_expert, seg_offsets, seg_first_rank, dest, src, xp,
                                 status, ws, stream=None):
    """Testing only: a dispatch whose look-back waits cannot end; they time out (see the header)."""
    _check("moe_testing_dispatch_stalled", load_library().moe_testing_dispatch_stalled(
        ctypes.byref(s), _ptr(x), _ptr(topk_ids), _ptr(counts), _ptr(seg_expert), _ptr(seg_offsets),
        _ptr(seg_first_rank), _ptr(dest), _ptr(src), _ptr(xp), _ptr(status), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_expert_gate_up(s, xp, seg_expert, seg_offsets, w_gate, w_up, hp, status=None, stream=None):
    _check("moe_expert_gate_up", load_library().moe_expert_gate_up(
        ctypes.byref(s), _ptr(xp), _ptr(seg_expert), _ptr(seg_offsets), _ptr(w_gate), _ptr(w_up), _ptr(hp),
        _ptr(status), _stream(stream)))


def moe_testing_reroute_stalled(s, x, topk_ids, logits, counts, seg_expert, seg_offsets, seg_first_rank, dest, src,
                                xp, status, ws, stream=None):
    """Testing only: the re-routing dispatch with CTA 0 never arriving at the first grid barrier."""
    _check("moe_testing_reroute_stalled", load_library().moe_testing_reroute_stalled(
        ctypes.byref(s), _ptr(x), _ptr(topk_ids), _ptr(logits), _ptr(counts), _ptr(seg_expert), _ptr(seg_offsets),
        _ptr(seg_first_rank), _ptr(dest), _ptr(src), _ptr(xp), _ptr(status), _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_testing_gemm_stalled(s, xp, seg_expert, seg_offsets, w_gate, w_up, hp, status, stream=None):
    """Testing only: a gate/up GEMM whose first pipeline stage is never filled; its waits time out."""
    _check("moe_testing_gemm_stalled", load_library().moe_testing_gemm_stalled(
        ctypes.byref(s), _ptr(xp), _ptr(seg_expert), _ptr(seg_offsets), _ptr(w_gate), _ptr(w_up), _ptr(hp),
        _ptr(status), _stream(stream)))


def moe_expert_down(s, hp, seg_expert, seg_offsets, w_down, yp, status=None, stream=None):
    _check("moe_expert_down", load_library().moe_expert_down(
        ctypes.byref(s), _ptr(hp), _ptr(seg_expert), _ptr(seg_offsets), _ptr(w_down), _ptr(yp), _ptr(status),
        _stream(stream)))


def moe_expert_ffn(s, xp, seg_expert, seg_offsets, w_gate, w_up, w_down, hp, yp, status=None, stream=None):
    _check("moe_expert_ffn", load_library().moe_expert_ffn(
        ctypes.byref(s), _ptr(xp), _ptr(seg_expert), _ptr(seg_offsets), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
        _ptr(hp), _ptr(yp), _ptr(status), _stream(stream)))


def moe_combine(s, yp, dest, topk_w, out, stream=None):
    _check("moe_combine", load_library().moe_combine(
        ctypes.byref(s), _ptr(yp), _ptr(dest), _ptr(topk_w), _ptr(out), _stream(stream)))


def moe_combine_add(s, yp, dest, topk_w, base, out, stream=None):
    _check("moe_combine_add", load_library().moe_combine_add(
        ctypes.byref(s), _ptr(yp), _ptr(dest), _ptr(topk_w), _ptr(base), _ptr(out), _stream(stream)))


def moe_shared_expert(s, d_ff_shared, x, w_gate_s, w_up_s, w_down_s, h_s, y_s, status=None, stream=None):
    _check("moe_shared_expert", load_library().moe_shared_expert(
        ctypes.byref(s), int(d_ff_shared), _ptr(x), _ptr(w_gate_s), _ptr(w_up_s), _ptr(w_down_s), _ptr(h_s),
        _ptr(y_s), _ptr(status), _stream(stream)))


def moe_layer_fwd(s, x, w_router, bias, w_gate, w_up, w_down, out, status, ws, stream=None):
    _check("moe_layer_fwd", load_library().moe_layer_fwd(
        ctypes.byref(s), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(out),
        _ptr(status), _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def moe_layer_fwd_aux(s, x, w_router, bias, w_gate, w_up, w_down, out, status, ws, topk_ids=None, topk_w=None,
                      counts=None, seg_offsets=None, dest=None, stats=None, stream=None):
    """moe_layer_fwd plus the routing results copied into the given tensors (None = not wanted)."""
    aux = MoeAux(_ptr(topk_ids), _ptr(topk_w), _ptr(counts), _ptr(seg_offsets), _ptr(dest), _ptr(stats))
    _check("moe_layer_fwd_aux", load_library().moe_layer_fwd_aux(
        ctypes.byref(s), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(out),
        ctypes.byref(aux), _ptr(status), _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_layer_views(s, ws) -> MoeLayerViews:
    v = MoeLayerViews()
    _check("moe_layer_views", load_library().moe_layer_views(ctypes.byref(s), _ptr(ws), ctypes.byref(v)))
    return v


def moe_route_scores(s, x, w_router, bias, scores, status=None, stream=None):
    _check("moe_route_scores", load_library().moe_route_scores(
        ctypes.byref(s), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(scores), _ptr(status), _stream(stream)))


def moe_expert_choose(s, scores, x, seg_expert, seg_offsets, src, row_w, emap, xp, stream=None):
    _check("moe_expert_choose", load_library().moe_expert_choose(
        ctypes.byref(s), _ptr(scores), _ptr(x), _ptr(seg_expert), _ptr(seg_offsets), _ptr(src), _ptr(row_w),
        _ptr(emap), _ptr(xp), _stream(stream)))


def moe_combine_expert_choice(s, yp, emap, row_w, base, out, stream=None):
    _check("moe_combine_expert_choice", load_library().moe_combine_expert_choice(
        ctypes.byref(s), _ptr(yp), _ptr(emap), _ptr(row_w), _ptr(base), _ptr(out), _stream(stream)))


def moe_route_workspace_size(s) -> int:
    n = ctypes.c_size_t()
    _check("moe_route_workspace_size", load_library().moe_route_workspace_size(ctypes.byref(s), ctypes.byref(n)))
    return n.value


def _nbytes(ws):
    return ws.numel() * ws.element_size() if ws is not None else 0


def moe_route_ws(s, x, w_router, bias, logits, topk_ids, topk_w, status=None, ws=None, stream=None):
    _check("moe_route_ws", load_library().moe_route_ws(
        ctypes.byref(s), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(logits), _ptr(topk_ids), _ptr(topk_w),
        _ptr(status), _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_route_scores_ws(s, x, w_router, bias, scores, status=None, ws=None, stream=None):
    _check("moe_route_scores_ws", load_library().moe_route_scores_ws(
        ctypes.byref(s), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(scores), _ptr(status), _ptr(ws), _nbytes(ws),
        _stream(stream)))


def moe_dispatch_reroute(s, x, topk_ids, logits, counts, seg_expert, seg_offsets, seg_first_rank, dest, src, xp,
                         status=None, ws=None, stream=None):
    _check("moe_dispatch_reroute", load_library().moe_dispatch_reroute(
        ctypes.byref(s), _ptr(x), _ptr(topk_ids), _ptr(logits), _ptr(counts), _ptr(seg_expert), _ptr(seg_offsets),
        _ptr(seg_first_rank), _ptr(dest), _ptr(src), _ptr(xp), _ptr(status), _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_routing_stats(s, counts, seg_expert, seg_offsets, stats, stream=None):
    """stats: int32 CUDA tensor of len(STAT_NAMES) values (see the header for their meaning)."""
    _check("moe_routing_stats", load_library().moe_routing_stats(
        ctypes.byref(s), _ptr(counts), _ptr(seg_expert), _ptr(seg_offsets), _ptr(stats), _stream(stream)))


# ----------------------------------------------------------------------------- expert parallelism

EP_MAX_RANKS = 16


def _ptr_table(tensors):
    """A host array of device pointers (entry i = tensors[i]'s address), as the moe_ep_* calls take."""
    return (ctypes.c_void_p * len(tensors))(*[_ptr(t) for t in tensors])


def moe_ep_sizes(s):
    """(xp_bytes, replica_weight_bytes, n_local_segments) of one rank."""
    a, b, n = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_int32()
    _check("moe_ep_sizes", load_library().moe_ep_sizes(ctypes.byref(s), ctypes.byref(a), ctypes.byref(b),
                                                        ctypes.byref(n)))
    return a.value, b.value, n.value


def moe_ep_plan(s, rank, counts_all, counts, seg_expert, seg_slot, seg_offsets, status=None, stream=None):
    _check("moe_ep_plan", load_library().moe_ep_plan(
        ctypes.byref(s), int(rank), _ptr(counts_all), _ptr(counts), _ptr(seg_expert), _ptr(seg_slot),
        _ptr(seg_offsets), _ptr(status), _stream(stream)))


def moe_ep_prefetch_weights(s, rank, seg_expert, seg_offsets, w_gate, w_up, w_down, stream=None):
    """w_gate / w_up / w_down: lists of R tensors (every rank's weight slots; entry `rank` is written)."""
    _check("moe_ep_prefetch_weights", load_library().moe_ep_prefetch_weights(
        ctypes.byref(s), int(rank), _ptr(seg_expert), _ptr(seg_offsets), _ptr_table(w_gate), _ptr_table(w_up),
        _ptr_table(w_down), _stream(stream)))


def moe_ep_dispatch(s, src_rank, x, topk_ids, counts_all, dest, xp, src, status=None, stream=None):
    """x / topk_ids / dest: lists of the n_src source ranks' tensors; xp / src: lists of R owners' buffers."""
    _check("moe_ep_dispatch", load_library().moe_ep_dispatch(
        ctypes.byref(s), int(src_rank), len(x), _ptr_table(x), _ptr_table(topk_ids), _ptr(counts_all),
        _ptr_table(dest), _ptr_table(xp), _ptr_table(src), _ptr(status), _stream(stream)))


def moe_ep_expert_ffn(s, xp, seg_slot, seg_offsets, w_gate, w_up, w_down, hp, yp, status=None, stream=None):
    _check("moe_ep_expert_ffn", load_library().moe_ep_expert_ffn(
        ctypes.byref(s), _ptr(xp), _ptr(seg_slot), _ptr(seg_offsets), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
        _ptr(hp), _ptr(yp), _ptr(status), _stream(stream)))


def moe_ep_combine(s, src_rank, yp, dest, topk_w, out, stream=None):
    """yp: list of R owners' Yp; dest / topk_w / out: lists of the n_src source ranks' tensors."""
    _check("moe_ep_combine", load_library().moe_ep_combine(
        ctypes.byref(s), int(src_rank), len(dest), _ptr_table(yp), _ptr_table(dest), _ptr_table(topk_w),
        _ptr_table(out), _stream(stream)))
