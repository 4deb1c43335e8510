"""Plain, slow fp64 CPU oracle of the top-k MoE FFN layer forward.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or call anything in
this package.  The CUDA library never calls it, and it shares no code with
the CUDA library; both only take their inputs from the seeded generator
module ``mixture_experts_routing_02_b200.synthetic``.

Sources (web pages; section names are the pages' own headings):

* [MoE-impl] "Sparsely-Gated MoE 구현 관점에서 살펴보기: Router, Top-k, 부하 분산"
  (molayo1419.me).  Sections used: "Router를 텐서 형태에서 추적하기" (shapes),
  "Top-2 라우팅의 수치 예시" (worked top-2 example), "순전파 과정(forward pass)은
  디스패치와 결합(combine)을 포함" (the forward pipeline), "로드 밸런싱 손실(load-balancing loss)과
  용량(capacity)은 별개" (capacity and overflow), "pure Python으로 Top-k Router
  확인하기" (stable softmax over the selected logits).
* [MoonEP] "가장 바쁜 랭크가 속도를 정합니다: MoonEP의 계획 코드를 직접 돌려봤습니다"
  (thakicloud.com).  Sections "개요", "이 기술은 무엇인가", "설치 및 통합",
  "실제 실험 결과" (balanced plan: exactly S x K rows per rank, replica slots,
  cu_seqlens, the CAP check).
* [EP-textbook] "5.3 Expert Parallelism (전문가 병렬화)" (sungeuns.github.io),
  section "2. 디스패처 엔지니어링" (per-destination bincount) and
  "3. 고도화된 최적화: 오버래핑(Overlapping) 및 GroupGEMM" (grouped expert GEMM).
* [Token-skew] "Expert를 똑같이 나눴는데도 GPU가 대기하는 이유: MoE의 토큰 쏠림"
  (portfolio.ywsung.com), the eager per-expert backend and the 8-expert /
  4-GPU skew example.

Everything is computed in float64 from the exact values of the bf16 / fp32
inputs, with no intermediate rounding, except where a floating-point value
decides an integer (the top-k selection): that decision is taken on the
logits rounded to fp32, the precision the kernels decide in.

Readings where the pages are silent or garbled:
ties in the top-k go to the lower expert id; rows of one expert are ordered
by the flat index q = t*k + j; capacity C = ceil(cf * T * k / E); a dropped
(t, j) contributes nothing and the kept weights are not renormalised; the
router bias is added before selection and softmax; the balanced plan is the
deterministic greedy of ``balanced_plan``.

Parity status: every function here is pinned by tests in
``tests/test_oracle_pins.py`` (worked example, brute force, closed forms,
library routines, invariants); none is "parity unpinned" except the
comparison with the MoonEP page's table values at sigma > 0, which the
oracle does not try to reproduce (their generator is not published).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np


# ----------------------------------------------------------------------------
# conversions
# ----------------------------------------------------------------------------

def f64(a) -> np.ndarray:
    """Exact float64 copy of a torch tensor (bf16/fp32) or a numpy array."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        import torch  # local: numpy-only callers need no torch
        if a.dtype in (torch.bfloat16, torch.float16):
            a = a.to(torch.float32)
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


def i64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.asarray(a, dtype=np.int64)


# ----------------------------------------------------------------------------
# step 1: router logits   [MoE-impl] "순전파 과정 ..." first bullet: X @ W_r.T
# ----------------------------------------------------------------------------

def router_logits(x, w_router, bias=None) -> np.ndarray:
    """logits[t, e] = sum_i x[t, i] * w_r[e, i] + b[e]   (fp64, [T, E]).

    Shapes follow [MoE-impl] "Router를 텐서 형태에서 추적하기": X [T, d],
    W_r [E, d] (the page writes the projection as X @ W_r.T).
    """
    logits = f64(x) @ f64(w_router).T
    if bias is not None:
        logits = logits + f64(bias)[None, :]
    return logits


# ----------------------------------------------------------------------------
# step 2-3: top-k and renormalised softmax   [MoE-impl] "Top-2 라우팅의 수치 예시"
# ----------------------------------------------------------------------------

def topk_ids(logits64: np.ndarray, k: int) -> np.ndarray:
    """ids[t, 0..k-1]: the k largest logits of row t in descending order.

    The comparison is made on the logits rounded to fp32 (the precision the
    kernels decide in); equal values go to the lower expert id.  A stable
    sort of the negated values gives exactly that order.
    """
    l32 = np.asarray(logits64, dtype=np.float64).astype(np.float32)
    order = np.argsort(-l32, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def topk_weights(logits64: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """w[t, j] = exp(l_j - l_max) / sum_{j' selected} exp(l_j' - l_max).

    Softmax over the selected logits only, shifted by their maximum so the
    exponent cannot overflow ([MoE-impl] "pure Python으로 Top-k Router
    확인하기").  This equals a softmax over all E experts followed by
    renormalisation over the selected k, so the two orders the page mentions
    give the same weights.
    """
    sel = np.take_along_axis(np.asarray(logits64, dtype=np.float64), ids, axis=1)
    m = sel.max(axis=1, keepdims=True)
    e = np.exp(sel - m)
    return e / e.sum(axis=1, keepdims=True)


def topk_weights_softmax_all(logits64: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """The other order the page mentions, without renormalisation: a softmax over all E
    logits, read at the selected experts (the k weights sum to less than 1)."""
    l = np.asarray(logits64, dtype=np.float64)
    e = np.exp(l - l.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)
    return np.take_along_axis(p, ids, axis=1)


def route(x, w_router, bias, k: int, softmax_all: bool = False):
    """(logits fp64 [T,E], ids int64 [T,k], weights fp64 [T,k])."""
    logits = router_logits(x, w_router, bias)
    ids = topk_ids(logits, k)
    w = topk_weights_softmax_all(logits, ids) if softmax_all else topk_weights(logits, ids)
    return logits, ids, w


# ----------------------------------------------------------------------------
# step 4: histogram   [EP-textbook] "2. 디스패처 엔지니어링" (bincount);
#                     [MoonEP] "설치 및 통합" (tokens_per_expert [E] int32)
# ----------------------------------------------------------------------------

def histogram(ids: np.ndarray, E: int) -> np.ndarray:
    counts = np.zeros(E, dtype=np.int64)
    for e in i64(ids).ravel():
        counts[e] += 1
    return counts


# ----------------------------------------------------------------------------
# step 5: stable rank of each (t, j) inside its expert
# ----------------------------------------------------------------------------

def expert_rank(ids: np.ndarray, E: int) -> np.ndarray:
    """rank[q] = number of q' < q (q = t*k + j) routed to the same expert."""
    flat = i64(ids).ravel()
    seen = np.zeros(E, dtype=np.int64)
    rank = np.empty(flat.size, dtype=np.int64)
    for q, e in enumerate(flat):
        rank[q] = seen[e]
        seen[e] += 1
    return rank


# ----------------------------------------------------------------------------
# step 6: capacity   [MoE-impl] "로드 밸런싱 손실(load-balancing loss)과 용량(capacity)은 별개"
# ----------------------------------------------------------------------------

def capacity_rows(capacity_factor: float, T: int, k: int, E: int) -> int:
    """C = ceil(cf * T * k / E); 0 means no limit (cf == 0).

    The page's formula did not survive extraction; this is the usual
    capacity-factor form of the GShard / Switch line the page cites.
    """
    if capacity_factor <= 0:
        return 0
    return int(math.ceil(capacity_factor * T * k / E))


# ----------------------------------------------------------------------------
# segments: the expert-contiguous layout of the dispatched rows
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Segments:
    expert: np.ndarray      # [n_seg] expert of each segment (-1 = unused slot)
    length: np.ndarray      # [n_seg] rows in each segment
    first_rank: np.ndarray  # [n_seg] within-expert rank of the segment's first row

    @property
    def offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.length)]).astype(np.int64)


def plain_segments(counts: np.ndarray, capacity: int = 0) -> Segments:
    """One segment per expert, in expert order, holding min(count, C) rows."""
    E = len(counts)
    length = np.array([min(c, capacity) if capacity > 0 else c for c in counts], dtype=np.int64)
    return Segments(expert=np.arange(E, dtype=np.int64), length=length,
                    first_rank=np.zeros(E, dtype=np.int64))


class PlanInfeasible(Exception):
    """More replica pieces than replica slots in one group (the CAP check)."""


@dataclasses.dataclass
class PlanStats:
    loads: np.ndarray        # [R] rows homed in each group before planning
    migrated_rows: int       # rows served outside their home group
    replicas_used: int       # replica slots holding a piece


def balanced_plan(counts: np.ndarray, R: int, S: int, k: int, B: int) -> Tuple[Segments, PlanStats]:
    """Replicate overloaded experts so each of R groups gets exactly S*k rows.

    What the MoonEP page fixes ("개요", "이 기술은 무엇인가", "설치 및 통합",
    "실제 실험 결과"): experts are homed contiguously, E/R per group; every
    group receives exactly S*K rows; overflowing experts get copies in the
    spare slots [E, E+B) of other groups; a plan whose allocation exceeds the
    capacity is an error.  The planning algorithm itself is not given; this
    deterministic greedy is the reading used here:

    1. CAP = S*k, home(e) = e // (E/R), load[g] = sum of counts homed in g.
    2. Groups above CAP, in ascending order, give up load[g] - CAP rows,
       taken from their experts in descending count (ties: lower id); each
       expert gives min(count, rows still to give).  These (expert, rows)
       chunks form one queue in that order.
    3. Groups below CAP, in ascending order, take CAP - load[g] rows from the
       front of the queue, splitting chunks where needed; each (expert, group)
       piece occupies the group's next replica slot.  More than B pieces in a
       group raises PlanInfeasible.
    4. An expert's rows (in stable q order) fill its home segment first
       (count - given rows), then its pieces in creation order.
    5. Group g lays out its home experts in ascending id, then its B replica
       slots in creation order (unused slots: expert -1, 0 rows).
    """
    counts = i64(counts)
    E = len(counts)
    if E % R != 0:
        raise ValueError("E must be a multiple of R")
    epg = E // R
    CAP = S * k
    if int(counts.sum()) != R * CAP:
        raise ValueError("sum(counts) must equal R*S*k")

    loads = np.array([int(counts[g * epg:(g + 1) * epg].sum()) for g in range(R)], dtype=np.int64)
    given = np.zeros(E, dtype=np.int64)
    queue: List[List[int]] = []
    for g in range(R):
        excess = int(loads[g]) - CAP
        if excess <= 0:
            continue
        members = sorted(range(g * epg, (g + 1) * epg), key=lambda e: (-int(counts[e]), e))
        for e in members:
            if excess == 0:
                break
            take = min(int(counts[e]), excess)
            if take > 0:
                given[e] = take
                queue.append([e, take])
                excess -= take

    slots: Dict[int, List[Tuple[int, int]]] = {g: [] for g in range(R)}
    head = 0
    for g in range(R):
        deficit = CAP - int(loads[g])
        while deficit > 0:
            e, avail = queue[head]
            take = min(avail, deficit)
            slots[g].append((e, take))
            queue[head][1] -= take
            deficit -= take
            if queue[head][1] == 0:
                head += 1
        if len(slots[g]) > B:
            raise PlanInfeasible(f"group {g} needs {len(slots[g])} replica slots > B={B}")

    # within-expert rank at which each piece starts, in creation order
    next_rank = {e: int(counts[e] - given[e]) for e in range(E)}
    seg_e, seg_n, seg_r = [], [], []
    for g in range(R):
        for e in range(g * epg, (g + 1) * epg):
            seg_e.append(e)
            seg_n.append(int(counts[e] - given[e]))
            seg_r.append(0)
        for i in range(B):
            if i < len(slots[g]):
                e, n = slots[g][i]
                seg_e.append(e)
                seg_n.append(n)
                seg_r.append(next_rank[e])
                next_rank[e] += n
            else:
                seg_e.append(-1)
                seg_n.append(0)
                seg_r.append(0)
    segs = Segments(expert=np.array(seg_e, dtype=np.int64), length=np.array(seg_n, dtype=np.int64),
                    first_rank=np.array(seg_r, dtype=np.int64))
    stats = PlanStats(loads=loads, migrated_rows=int(given.sum()),
                      replicas_used=int(sum(len(v) for v in slots.values())))
    return segs, stats


def num_segments(E: int, R: int, B: int) -> int:
    return E if R == 0 else R * (E // R + B)


# ----------------------------------------------------------------------------
# step 7: dispatch (final-slot positions and the permuted rows)
#   [MoE-impl] "순전파 과정 ..." (permute tokens into expert order);
#   [MoonEP] "이 기술은 무엇인가" (each row is written straight to its final slot)
# ----------------------------------------------------------------------------

def dispatch_positions(ids: np.ndarray, segs: Segments, E: int):
    """dest[q] (row of pair q in the dispatched buffer, -1 if dropped) and src[row] = q."""
    flat = i64(ids).ravel()
    rank = expert_rank(ids, E)
    offsets = segs.offsets
    pieces: Dict[int, List[int]] = {}
    for s, e in enumerate(segs.expert):
        if e >= 0:
            pieces.setdefault(int(e), []).append(s)
    dest = np.full(flat.size, -1, dtype=np.int64)
    for q, e in enumerate(flat):
        r = rank[q]
        for s in pieces.get(int(e), []):
            r0 = segs.first_rank[s]
            if r0 <= r < r0 + segs.length[s]:
                dest[q] = offsets[s] + (r - r0)
                break
    rows = int(offsets[-1])
    src = np.full(rows, -1, dtype=np.int64)
    for q in range(flat.size):
        if dest[q] >= 0:
            src[dest[q]] = q
    return dest, src


def permute_rows(x, src: np.ndarray, k: int) -> np.ndarray:
    """Xp[row] = X[src[row] // k] (exact copy of the bf16 values, as fp64)."""
    x64 = f64(x)
    return x64[i64(src) // k]


# ----------------------------------------------------------------------------
# step 9: expert FFN (gated, three projections, SwiGLU)
#   [MoonEP] "설치 및 통합" (gate / up / down weights);
#   [EP-textbook] "3. ... GroupGEMM" (each expert's rows in one GEMM)
# ----------------------------------------------------------------------------

def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def expert_ffn(x_rows64: np.ndarray, w_gate_e, w_up_e, w_down_e):
    """(h, y) with h = silu(x W_g^T) * (x W_u^T) and y = h W_d^T, fp64, no rounding."""
    wg, wu, wd = f64(w_gate_e), f64(w_up_e), f64(w_down_e)
    h = silu(x_rows64 @ wg.T) * (x_rows64 @ wu.T)
    return h, h @ wd.T


def grouped_expert_ffn(xp64: np.ndarray, segs: Segments, w_gate, w_up, w_down):
    """Run every segment's rows through its expert: Hp [rows, F], Yp [rows, d]."""
    rows = xp64.shape[0]
    F = w_gate.shape[1]
    d = w_down.shape[1]
    hp = np.zeros((rows, F))
    yp = np.zeros((rows, d))
    off = segs.offsets
    for s, e in enumerate(segs.expert):
        if e < 0 or segs.length[s] == 0:
            continue
        a, b = off[s], off[s + 1]
        hp[a:b], yp[a:b] = expert_ffn(xp64[a:b], w_gate[e], w_up[e], w_down[e])
    return hp, yp


# ----------------------------------------------------------------------------
# step 10: combine   [MoE-impl] "순전파 과정 ..." last bullet (un-permute and
#                    weight by the router); [MoonEP] "설치 및 통합" (combine)
# ----------------------------------------------------------------------------

def combine(yp64: np.ndarray, dest: np.ndarray, weights64: np.ndarray, T: int, k: int) -> np.ndarray:
    """out[t] = sum over kept j of w[t, j] * y[dest[t*k + j]]."""
    d = yp64.shape[1]
    out = np.zeros((T, d))
    dest = i64(dest).reshape(T, k)
    for t in range(T):
        for j in range(k):
            r = dest[t, j]
            if r >= 0:
                out[t] += weights64[t, j] * yp64[r]
    return out


# ----------------------------------------------------------------------------
# the whole layer
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class LayerResult:
    logits: np.ndarray
    ids: np.ndarray
    weights: np.ndarray
    counts: np.ndarray
    segs: Segments
    dest: np.ndarray
    src: np.ndarray
    xp: np.ndarray
    hp: np.ndarray
    yp: np.ndarray
    out: np.ndarray
    plan: Optional[PlanStats] = None


def shared_expert(x, w_gate_s, w_up_s, w_down_s) -> np.ndarray:
    """The shared expert: one dense SwiGLU FFN applied to every token (fp64).

    [EP-textbook] "3. 고도화된 최적화: 오버래핑(Overlapping) 및 GroupGEMM", first optimisation:
    alongside the routed experts, one shared expert processes every token; its output is
    added to the routed combine.
    """
    return expert_ffn(f64(x), w_gate_s, w_up_s, w_down_s)[1]


def layer_forward(x, w_router, bias, w_gate, w_up, w_down, k: int,
                  capacity: int = 0, n_groups: int = 0, replica_slots: int = 0, shared=None,
                  softmax_all: bool = False) -> LayerResult:
    """Router -> top-k -> (capacity | balanced plan) -> dispatch -> expert FFN -> combine
    (+ the shared expert's output when ``shared`` = (W_gate_s, W_up_s, W_down_s))."""
    T = x.shape[0]
    E = w_router.shape[0]
    logits, ids, w = route(x, w_router, bias, k, softmax_all)
    counts = histogram(ids, E)
    plan = None
    if n_groups > 0:
        if capacity > 0:
            raise ValueError("capacity and the balanced plan exclude each other")
        segs, plan = balanced_plan(counts, n_groups, T // n_groups, k, replica_slots)
    else:
        segs = plain_segments(counts, capacity)
    dest, src = dispatch_positions(ids, segs, E)
    xp = permute_rows(x, src, k)
    hp, yp = grouped_expert_ffn(xp, segs, w_gate, w_up, w_down)
    out = combine(yp, dest, w, T, k)
    if shared is not None:
        out = out + shared_expert(x, *shared)
    return LayerResult(logits, ids, w, counts, segs, dest, src, xp, hp, yp, out, plan)


def token_output(x_row64: np.ndarray, ids_row: Sequence[int], w_row: Sequence[float],
                 w_gate, w_up, w_down, keep: Optional[Sequence[bool]] = None) -> np.ndarray:
    """One token's layer output evaluated directly, expert by expert (no dispatch)."""
    out = np.zeros(w_down.shape[1])
    for j, e in enumerate(ids_row):
        if keep is not None and not keep[j]:
            continue
        _, y = expert_ffn(x_row64[None, :], w_gate[int(e)], w_up[int(e)], w_down[int(e)])
        out += w_row[j] * y[0]
    return out


# ----------------------------------------------------------------------------
# inputs: the top-k margin rule (redraw rows of X whose top-(k+1) logits are too close)
# ----------------------------------------------------------------------------

def margin_violations(logits64: np.ndarray, k: int, min_gap: float) -> np.ndarray:
    """Rows whose consecutive gaps among the top-(k+1) logits fall below min_gap."""
    E = logits64.shape[1]
    m = min(k + 1, E)
    top = -np.sort(-logits64, axis=1)[:, :m]
    if m < 2:
        return np.zeros(logits64.shape[0], dtype=bool)
    gaps = top[:, :-1] - top[:, 1:]
    return (gaps < min_gap).any(axis=1)


def enforce_margin(x, w_router, bias, k: int, redraw, min_gap: float = 1e-3,
                   max_attempts: int = 1000):
    """Replace rows of X (a bf16 torch tensor, edited in place) until every
    token's top-(k+1) logits are at least min_gap apart.

    ``redraw(t, attempt)`` returns a new bf16 row; it comes from the seeded
    generator.  Returns the number of rows that were redrawn.
    """
    logits = router_logits(x, w_router, bias)
    bad = np.nonzero(margin_violations(logits, k, min_gap))[0]
    w64 = f64(w_router)
    b64 = f64(bias) if bias is not None else 0.0
    for t in bad:
        for attempt in range(max_attempts):
            row = redraw(int(t), attempt)
            lrow = f64(row)[None, :] @ w64.T + b64
            if not margin_violations(lrow, k, min_gap)[0]:
                x[int(t)] = row
                break
        else:
            raise RuntimeError(f"could not satisfy the top-k margin for token {t}")
    return len(bad)


# ----------------------------------------------------------------------------
# expert-choice routing   [Token-skew] "라우팅 분포와 학습 안정성": instead of tokens
# choosing experts, experts choose tokens
# ----------------------------------------------------------------------------

def expert_scores(logits64: np.ndarray) -> np.ndarray:
    """S[t, e]: softmax of token t's logits over the E experts (fp64)."""
    l = np.asarray(logits64, dtype=np.float64)
    e = np.exp(l - l.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


@dataclasses.dataclass
class ExpertChoice:
    scores: np.ndarray     # [T, E] fp64
    picks: List[np.ndarray]  # per expert: picked tokens, ascending id
    segs: Segments         # E segments of min(C, T) rows, expert order
    src: np.ndarray        # [rows] token of each dispatched row
    row_w: np.ndarray      # [rows] score S[t, e] of each row


def expert_choice(logits64: np.ndarray, capacity: int) -> ExpertChoice:
    """Each expert e takes the C tokens with the largest S[t, e] (compared in fp32, the
    kernels' precision; equal scores go to the lower token id); its segment lists them in
    ascending token order."""
    return select_tokens(expert_scores(logits64), capacity)


def select_tokens(S: np.ndarray, capacity: int) -> ExpertChoice:
    """The expert-choice selection on given scores S [T, E]."""
    S = np.asarray(S, dtype=np.float64)
    T, E = S.shape
    C = min(capacity, T)
    s32 = S.astype(np.float32)
    picks = []
    for e in range(E):
        order = np.argsort(-s32[:, e], kind="stable")[:C]
        picks.append(np.sort(order).astype(np.int64))
    length = np.full(E, C, dtype=np.int64)
    segs = Segments(expert=np.arange(E, dtype=np.int64), length=length, first_rank=np.zeros(E, dtype=np.int64))
    src = np.concatenate(picks) if E else np.zeros(0, dtype=np.int64)
    row_w = np.concatenate([S[picks[e], e] for e in range(E)]) if E else np.zeros(0)
    return ExpertChoice(S, picks, segs, src, row_w)


def expert_choice_forward(x, w_router, bias, w_gate, w_up, w_down, capacity: int):
    """out[t] = sum over the experts e that picked t of S[t, e] * FFN_e(x_t)."""
    logits = router_logits(x, w_router, bias)
    ec = expert_choice(logits, capacity)
    xp = f64(x)[ec.src]
    hp, yp = grouped_expert_ffn(xp, ec.segs, w_gate, w_up, w_down)
    out = combine_expert_choice(yp, ec.src, ec.row_w, f64(x).shape[0])
    return logits, ec, xp, hp, yp, out


def combine_expert_choice(yp64, src, row_w, T: int) -> np.ndarray:
    """out[t] = sum over the rows r with src[r] = t of row_w[r] * Yp[r] (rows in order)."""
    yp64 = np.asarray(yp64, dtype=np.float64)
    out = np.zeros((T, yp64.shape[1]))
    for r in range(len(src)):
        out[src[r]] += row_w[r] * yp64[r]
    return out


def expert_choice_map(ec: "ExpertChoice", T: int) -> np.ndarray:
    """[T, E] row of (t, e), or -1 where expert e did not keep token t."""
    E = len(ec.picks)
    m = np.full((T, E), -1, dtype=np.int64)
    for r in range(len(ec.src)):
        e = int(np.searchsorted(ec.segs.offsets, r, side="right") - 1)
        m[ec.src[r], e] = r
    return m


def ec_margin_violations(S: np.ndarray, capacity: int, min_rel_gap: float) -> np.ndarray:
    """Experts whose C-th and (C+1)-th largest scores are closer than min_rel_gap times the
    C-th, so that a rounding difference in the scores could change which tokens the expert
    keeps (a score's relative rounding error is about its logit's absolute error)."""
    S = np.asarray(S, dtype=np.float64)
    T, E = S.shape
    if capacity >= T:
        return np.zeros(E, dtype=bool)
    srt = -np.sort(-S, axis=0)
    return (srt[capacity - 1] - srt[capacity]) < min_rel_gap * srt[capacity - 1]


def enforce_ec_margin(x, w_router, bias, capacity: int, redraw, min_rel_gap: float = 5e-4,
                      max_redraws: int = 10000):
    """Replace rows of X (a bf16 torch tensor, edited in place) until every expert's C-th
    and (C+1)-th largest scores are at least min_rel_gap (relative) apart (``redraw(t,
    attempt)`` returns a new bf16 row from the seeded generator).  Returns the number of
    redraws."""
    logits = router_logits(x, w_router, bias)
    w64 = f64(w_router)
    b64 = f64(bias) if bias is not None else 0.0
    attempts = {}
    n = 0
    while True:
        S = expert_scores(logits)
        bad = np.nonzero(ec_margin_violations(S, capacity, min_rel_gap))[0]
        if len(bad) == 0:
            return n
        if n >= max_redraws:
            raise RuntimeError("could not satisfy the expert-choice margin")
        e = int(bad[0])
        t = int(np.argsort(-S[:, e], kind="stable")[capacity - 1])   # the last kept token
        a = attempts.get(t, 0)
        attempts[t] = a + 1
        row = redraw(t, a)
        x[t] = row
        logits[t] = f64(row) @ w64.T + b64
        n += 1


# ----------------------------------------------------------------------------
# overflow re-routing   [MoE-impl] "로드 밸런싱 손실(load-balancing loss)과 용량(capacity)은
# 별개": a pair over its expert's capacity may go to another candidate instead of being dropped
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Rerouted:
    expert: np.ndarray   # [T*k] final expert of each pair (-1: dropped for good)
    slot: np.ndarray     # [T*k] row of the pair inside its expert's segment
    round: np.ndarray    # [T*k] round in which the pair was placed (0: its own top-k expert)
    assigned: np.ndarray  # [E] rows of each expert (<= C)


def candidate_order(logits32_row: np.ndarray) -> List[int]:
    """A token's experts by logit, descending; equal logits: the lower id first."""
    return sorted(range(len(logits32_row)), key=lambda e: (-float(logits32_row[e]), e))


def reroute_overflow(ids: np.ndarray, logits64: np.ndarray, C: int) -> Rerouted:
    """Round 0: each expert keeps its first C pairs in q = t*k + j order (the capacity rule).
    Round r >= 1: every pair still unplaced proposes to its token's next candidate (in the
    token's logit order below its top-k, compared in fp32) among the experts that had room when
    the round began; a token's unplaced pairs take consecutive candidates in j order.  Each
    expert accepts the round's proposals in q order while it has room.  A pair with no
    candidate left is dropped.  Rows of a segment: round 0 pairs, then round 1, ... (q order
    inside a round)."""
    ids = i64(ids)
    T, k = ids.shape
    E = logits64.shape[1]
    l32 = np.asarray(logits64, dtype=np.float64).astype(np.float32)
    expert = np.full(T * k, -1, dtype=np.int64)
    slot = np.full(T * k, -1, dtype=np.int64)
    rnd = np.full(T * k, -1, dtype=np.int64)
    assigned = np.zeros(E, dtype=np.int64)
    pending = []
    for q in range(T * k):
        e = int(ids.ravel()[q])
        if assigned[e] < C:
            expert[q], slot[q], rnd[q] = e, assigned[e], 0
            assigned[e] += 1
        else:
            pending.append(q)
    order = {}      # token -> its candidates below the top-k, in logit order
    cursor = {}     # token -> next position in that list
    r = 0
    while pending:
        r += 1
        open_ = assigned < C
        if not open_.any():
            break
        proposals = []
        for q in pending:
            t = q // k
            if t not in order:
                held = set(int(e) for e in ids[t])
                order[t] = [e for e in candidate_order(l32[t]) if e not in held]
                cursor[t] = 0
            lst = order[t]
            while cursor[t] < len(lst) and not open_[lst[cursor[t]]]:
                cursor[t] += 1
            if cursor[t] < len(lst):
                proposals.append((q, lst[cursor[t]]))
                cursor[t] += 1
        room = C - assigned
        taken = np.zeros(E, dtype=np.int64)
        still = []
        for q, e in proposals:
            if taken[e] < room[e]:
                expert[q], slot[q], rnd[q] = e, assigned[e] + taken[e], r
                taken[e] += 1
            else:
                still.append(q)
        assigned += taken
        pending = still
    return Rerouted(expert, slot, rnd, assigned)


def reroute_positions(rr: Rerouted):
    """dest[q] and src[row] of the re-routed layout (one segment per expert)."""
    segs = Segments(expert=np.arange(len(rr.assigned), dtype=np.int64), length=rr.assigned.copy(),
                    first_rank=np.zeros(len(rr.assigned), dtype=np.int64))
    off = segs.offsets
    dest = np.where(rr.expert >= 0, off[np.maximum(rr.expert, 0)] + rr.slot, -1).astype(np.int64)
    src = np.full(int(off[-1]), -1, dtype=np.int64)
    for q in np.nonzero(dest >= 0)[0]:
        src[dest[q]] = q
    return segs, dest, src


def layer_forward_reroute(x, w_router, bias, w_gate, w_up, w_down, k: int, capacity: int):
    """The layer with overflow re-routing: a moved pair keeps its routing weight."""
    T = x.shape[0]
    logits, ids, w = route(x, w_router, bias, k)
    rr = reroute_overflow(ids, logits, capacity)
    segs, dest, src = reroute_positions(rr)
    xp = permute_rows(x, src, k)
    hp, yp = grouped_expert_ffn(xp, segs, w_gate, w_up, w_down)
    out = combine(yp, dest, w, T, k)
    return logits, ids, w, rr, segs, dest, src, xp, hp, yp, out
