"""Seeded synthetic inputs for the top-k MoE FFN layer forward.

This module only draws random numbers.  It holds none of the layer's
arithmetic: no router projection, no top-k, no softmax, no dispatch and no
expert FFN.  The CPU oracle (``oracle/``) and the CUDA path both take their
inputs from here, and nothing else is shared between them.

Workloads (shapes and value distributions follow the pages' workloads; the
pages' own models and benchmarks are not available, so these stand in):

* tiny            T=64     d=128  E=8   k=2 F=256
* mixtral-like    T=4096   d=4096 E=8   k=2 F=14336
* deepseek-like   T=4096   d=7168 E=256 k=8 F=2048
* skewed          T=8192   d=4096 E=64  k=2 F=1408, Zipf(1.2) router bias,
                  capacity factor 1.25 (tokens over capacity are dropped)
* balanced-plan   T=32768  d=7168 E=256 k=8 F=2048, Zipf(1.2) router bias,
                  R=8 virtual expert groups of S=4096 tokens, B=32 replica
                  slots per group
* expert-choice   the mixtral-like shape with expert-choice routing, each
                  expert keeping C = T*k/E = 1024 tokens
* expert-choice-e64  the skewed shape (Zipf(1.2) bias) with expert-choice
                  routing, C = 256 tokens per expert
* skewed-reroute  the skewed layer with overflow re-routed to other candidates

X ~ N(0, 1) and every weight ~ N(0, 0.02^2), drawn in fp32 and rounded to
bf16.  Each tensor (and each expert of an expert tensor) has its own
sub-seed derived from (seed, tensor name, index), so any piece can be
regenerated on its own.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Optional

import torch

WEIGHT_STD = 0.02


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    F: int
    zipf_s: float = 0.0            # 0 = no router bias
    capacity_factor: float = 0.0   # 0 = no capacity limit
    n_groups: int = 0              # R; 0 = no balanced plan
    replica_slots: int = 0         # B per group
    expert_choice: bool = False    # experts choose tokens; C = ceil(capacity_factor * T * k / E)
    reroute: bool = False          # pairs over capacity go to their token's next open candidate
    bf16_out: bool = False         # the full-size layer output meets the stated tolerance in bf16

    @property
    def tokens_per_group(self) -> int:
        return self.T // self.n_groups if self.n_groups else self.T

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


TINY = Workload("tiny", T=64, d=128, E=8, k=2, F=256)
MIXTRAL_LIKE = Workload("mixtral-like", T=4096, d=4096, E=8, k=2, F=14336, bf16_out=True)
DEEPSEEK_LIKE = Workload("deepseek-like", T=4096, d=7168, E=256, k=8, F=2048, bf16_out=True)
SKEWED = Workload("skewed", T=8192, d=4096, E=64, k=2, F=1408,
                  zipf_s=1.2, capacity_factor=1.25, bf16_out=True)
BALANCED = Workload("balanced-plan", T=32768, d=7168, E=256, k=8, F=2048,
                    zipf_s=1.2, n_groups=8, replica_slots=32)

# Expert-choice routing on the mixtral-like and skewed shapes: each expert keeps
# C = ceil(1.0 * T * k / E) tokens, so the experts' GEMMs have the rows of the top-k runs.
EXPERT_CHOICE = Workload("expert-choice", T=4096, d=4096, E=8, k=2, F=14336, capacity_factor=1.0,
                         expert_choice=True)
EXPERT_CHOICE_E64 = Workload("expert-choice-e64", T=8192, d=4096, E=64, k=2, F=1408, zipf_s=1.2,
                             capacity_factor=1.0, expert_choice=True)

# The skewed layer with its overflow re-routed instead of dropped.
SKEWED_REROUTE = Workload("skewed-reroute", T=8192, d=4096, E=64, k=2, F=1408, zipf_s=1.2, capacity_factor=1.25,
                          reroute=True)

# Reduced copies for profiling captures that must stay at a few GB on the device: the same
# per-expert shapes and rows per expert as the full workloads, with fewer experts.
DEEPSEEK_LIKE_E32 = Workload("deepseek-like-e32", T=512, d=7168, E=32, k=8, F=2048)
BALANCED_E32 = Workload("balanced-plan-e32", T=4096, d=7168, E=32, k=8, F=2048,
                        zipf_s=1.2, n_groups=2, replica_slots=16)

WORKLOADS = {w.name: w for w in (TINY, MIXTRAL_LIKE, DEEPSEEK_LIKE, SKEWED, BALANCED, DEEPSEEK_LIKE_E32,
                                 BALANCED_E32, EXPERT_CHOICE, EXPERT_CHOICE_E64, SKEWED_REROUTE)}


def sub_seed(seed: int, tag: str, *idx: int) -> int:
    """A 63-bit seed derived from (seed, tag, idx...) with BLAKE2b."""
    key = "/".join([str(int(seed)), tag] + [str(int(i)) for i in idx]).encode()
    return int.from_bytes(hashlib.blake2b(key, digest_size=8).digest(), "little") & ((1 << 63) - 1)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def zipf_bias(E: int, s: float) -> torch.Tensor:
    """Router bias b_e = ln p_e with p_e proportional to (e+1)^-s (expert 0 hottest)."""
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    p = ranks.pow(-s)
    p = p / p.sum()
    return p.log().to(torch.float32)


def router_inputs(w: Workload, seed: int = 0):
    """X [T, d] bf16, W_r [E, d] bf16 and the optional bias [E] fp32 (CPU tensors)."""
    x = torch.randn(w.T, w.d, generator=_gen("cpu", sub_seed(seed, "x"))).to(torch.bfloat16)
    w_r = (torch.randn(w.E, w.d, generator=_gen("cpu", sub_seed(seed, "w_router"))) * WEIGHT_STD
           ).to(torch.bfloat16)
    bias = zipf_bias(w.E, w.zipf_s) if w.zipf_s > 0 else None
    return x, w_r, bias


def x_row_redraw(w: Workload, seed: int, t: int, attempt: int) -> torch.Tensor:
    """Replacement row t of X for the given redraw attempt (bf16 [d])."""
    g = _gen("cpu", sub_seed(seed, "x-redraw", t, attempt))
    return torch.randn(w.d, generator=g).to(torch.bfloat16)


def expert_weights(w: Workload, seed: int = 0, device="cpu", experts: Optional[range] = None):
    """W_gate, W_up [E, F, d] and W_down [E, d, F], bf16, nn.Linear [out, in] layout.

    Each expert slice is drawn from its own generator on ``device``; the
    streams of a CUDA generator differ from a CPU generator's, so a workload
    must be generated on one device and copied.
    """
    experts = range(w.E) if experts is None else experts
    n = len(experts)
    wg = torch.empty(n, w.F, w.d, dtype=torch.bfloat16, device=device)
    wu = torch.empty(n, w.F, w.d, dtype=torch.bfloat16, device=device)
    wd = torch.empty(n, w.d, w.F, dtype=torch.bfloat16, device=device)
    for i, e in enumerate(experts):
        for name, dst, shape in (("w_gate", wg, (w.F, w.d)), ("w_up", wu, (w.F, w.d)),
                                 ("w_down", wd, (w.d, w.F))):
            g = _gen(device, sub_seed(seed, name, e))
            dst[i].copy_((torch.randn(shape, generator=g, device=device) * WEIGHT_STD)
                         .to(torch.bfloat16))
    return wg, wu, wd


def shared_expert_weights(w: Workload, d_ff_shared: int, seed: int = 0, device="cpu"):
    """The shared expert's W_gate, W_up [F_s, d] and W_down [d, F_s] (bf16)."""
    out = []
    for name, shape in (("ws_gate", (d_ff_shared, w.d)), ("ws_up", (d_ff_shared, w.d)), ("ws_down", (w.d, d_ff_shared))):
        g = _gen(device, sub_seed(seed, name))
        out.append((torch.randn(shape, generator=g, device=device) * WEIGHT_STD).to(torch.bfloat16))
    return tuple(out)


def lognormal_topk_ids(E: int, T: int, k: int, sigma: float, seed: int = 0) -> torch.Tensor:
    """Skewed routing ids [T, k] int32 drawn directly, without a router.

    Expert popularity is log p_e = sigma * z_e with z ~ N(0, 1); each token
    takes k distinct experts by perturbing log p with Gumbel noise and keeping
    the k largest (sampling without replacement in proportion to p).
    """
    z = torch.randn(E, generator=_gen("cpu", sub_seed(seed, "popularity")), dtype=torch.float64)
    logp = sigma * z
    u = torch.rand(T, E, generator=_gen("cpu", sub_seed(seed, "gumbel")), dtype=torch.float64)
    u = u.clamp_min(1e-300)
    keys = logp[None, :] - torch.log(-torch.log(u))
    return torch.topk(keys, k, dim=1).indices.to(torch.int32)


def uniform_roundrobin_ids(E: int, T: int, k: int) -> torch.Tensor:
    """ids[t, j] = (t*k + j) mod E: every expert receives T*k/E rows when E divides T*k."""
    q = torch.arange(T * k, dtype=torch.int64).reshape(T, k)
    return (q % E).to(torch.int32)


def gib(nbytes: float) -> float:
    return nbytes / float(1 << 30)


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = [
    "Workload", "TINY", "MIXTRAL_LIKE", "DEEPSEEK_LIKE", "SKEWED", "BALANCED", "DEEPSEEK_LIKE_E32", "BALANCED_E32",
    "EXPERT_CHOICE", "EXPERT_CHOICE_E64", "SKEWED_REROUTE",
    "WORKLOADS",
    "sub_seed", "zipf_bias", "router_inputs", "x_row_redraw", "expert_weights", "shared_expert_weights",
    "lognormal_topk_ids", "uniform_roundrobin_ids", "gib", "ceil_div",
]
