"""Seeded synthetic workloads for the FP8 x FP4 MoE expert layer.

This module only draws random numbers and holds the workload table.  It holds
none of the layer's arithmetic (no quantisation, no GEMM, no activation): the
CUDA library and the CPU oracle each quantise these bf16 draws themselves.

Recipe (the data-generation recipe of the DeepGEMM PR #416 review thread,
"_bf16_shared_worker" test body, restated; sizes from the workload table):

* activations ``x``: bf16 ``randn * 0.5`` of shape ``[T, H]``;
* per expert ``e``: ``L1[e]`` bf16 ``randn * 0.04`` of shape ``[2I, H]`` (rows
  ``0..I-1`` gate, ``I..2I-1`` up) and ``L2[e]`` bf16 ``randn * 0.04`` of shape
  ``[H, I]``;
* uniform routing: per token, the top-k of ``E`` uniform scores (k distinct
  experts, slot order = descending score); weights = softmax over the k slots of
  N(0,1) fp32 logits;
* skewed routing: the same, but the scores are Gumbel-perturbed log
  popularities, popularity of the expert at rank ``r`` of a seeded random
  expert order being ``1/(r+1)^s`` (Gumbel top-k = sampling k experts without
  replacement in proportion to popularity).

Every tensor is drawn from its own ``torch.Generator`` whose seed is derived
from ``(seed, tag, index)``, so any expert's weights can be regenerated alone
(the oracle needs only the experts a sampled token touches).  A generator on
``cuda`` gives different numbers than one on ``cpu`` for the same seed; callers
pick one device and hand the same bf16 tensors to both implementations.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    E: int
    k: int
    H: int
    I: int
    seed: int
    routing: str = "uniform"   # "uniform" | "zipf"
    zipf_s: float = 1.2

    @property
    def R(self) -> int:
        return self.T * self.k

    @property
    def flops(self) -> int:
        """2*T*k*3*H*I: GEMM1 (2I x H) plus GEMM2 (H x I) per routed row."""
        return 2 * self.T * self.k * 3 * self.H * self.I

    def asdict(self):
        return asdict(self)


# The five workloads: tiny parity case, decode, small batch, prefill, skewed prefill.
WORKLOADS = {
    0: Workload("tiny", T=64, E=8, k=2, H=256, I=256, seed=0),
    1: Workload("decode", T=8, E=384, k=6, H=7168, I=3072, seed=1),
    2: Workload("small", T=128, E=384, k=6, H=7168, I=3072, seed=2),
    3: Workload("prefill", T=8192, E=384, k=6, H=7168, I=3072, seed=3),
    4: Workload("skewed", T=4096, E=256, k=8, H=7168, I=2048, seed=4, routing="zipf", zipf_s=1.2),
}


def custom(name="custom", *, T, E, k, H, I, seed=0, routing="uniform", zipf_s=1.2) -> Workload:
    return Workload(name, T=T, E=E, k=k, H=H, I=I, seed=seed, routing=routing, zipf_s=zipf_s)


def _generator(device, seed: int, tag: str, index: int = 0) -> torch.Generator:
    digest = hashlib.sha256(f"{seed}/{tag}/{index}".encode()).digest()
    g = torch.Generator(device=device)
    g.manual_seed(int.from_bytes(digest[:8], "little") & ((1 << 63) - 1))
    return g


def _randn_bf16(shape, scale, device, seed, tag, index=0):
    g = _generator(device, seed, tag, index)
    return torch.randn(shape, dtype=torch.bfloat16, device=device, generator=g).mul_(scale)


def gen_x(w: Workload, device="cpu") -> torch.Tensor:
    """bf16 [T, H] activations, N(0, 0.5^2)."""
    return _randn_bf16((w.T, w.H), 0.5, device, w.seed, "x")


def gen_l1(w: Workload, e: int, device="cpu") -> torch.Tensor:
    """bf16 [2I, H] gate/up weights of expert e, N(0, 0.04^2)."""
    return _randn_bf16((2 * w.I, w.H), 0.04, device, w.seed, "l1", e)


def gen_l2(w: Workload, e: int, device="cpu") -> torch.Tensor:
    """bf16 [H, I] down-projection weights of expert e, N(0, 0.04^2)."""
    return _randn_bf16((w.H, w.I), 0.04, device, w.seed, "l2", e)


def gen_shared(T: int, SH: int, SI: int, seed: int, device="cpu"):
    """BF16 shared-expert inputs as the DeepGEMM PR #416 test body draws them:
    x [T, SH] ~ N(0, 0.25^2), L1 [2 SI, SH] and L2 [SH, SI] ~ N(0, 0.02^2)."""
    return (_randn_bf16((T, SH), 0.25, device, seed, "shared_x"),
            _randn_bf16((2 * SI, SH), 0.02, device, seed, "shared_l1"),
            _randn_bf16((SH, SI), 0.02, device, seed, "shared_l2"))


def gen_routing(w: Workload, device="cpu"):
    """(topk_idx int64 [T, k], topk_w fp32 [T, k]) as the recipe above states."""
    g = _generator(device, w.seed, "route")
    if w.routing == "uniform":
        scores = torch.rand((w.T, w.E), device=device, generator=g)
    elif w.routing == "zipf":
        order = torch.randperm(w.E, device=device, generator=g)
        ranks = torch.empty(w.E, dtype=torch.float64, device=device)
        ranks[order] = torch.arange(w.E, dtype=torch.float64, device=device)
        log_pop = -w.zipf_s * torch.log1p(ranks)
        u = torch.rand((w.T, w.E), dtype=torch.float64, device=device, generator=g)
        u = u.clamp_min(1e-300)
        scores = log_pop[None, :] - torch.log(-torch.log(u))
    else:
        raise ValueError(f"unknown routing {w.routing!r}")
    topk_idx = torch.topk(scores, w.k, dim=1, largest=True, sorted=True).indices.to(torch.int64)
    gl = _generator(device, w.seed, "logits")
    logits = torch.randn((w.T, w.k), dtype=torch.float32, device=device, generator=gl)
    topk_w = torch.softmax(logits, dim=1).contiguous()
    return topk_idx.contiguous(), topk_w


def structured_routing(T: int, k: int, E: int, device="cpu"):
    """The review thread's deterministic case: slot s of the flattened [T*k]
    index array goes to expert s % E, with unit weights."""
    idx = (torch.arange(T * k, dtype=torch.int64, device=device) % E).view(T, k)
    return idx.contiguous(), torch.ones((T, k), dtype=torch.float32, device=device)


def touched_experts(topk_idx: torch.Tensor, E: int):
    """Sorted list of valid expert ids that appear in topk_idx."""
    v = topk_idx.flatten()
    v = v[(v >= 0) & (v < E)]
    return sorted(set(int(e) for e in torch.unique(v).tolist()))
