"""Seeded synthetic inputs for the MXFP8 grouped expert MLP.

This module is shared by the CPU oracle, the GPU tests and the benchmark. It holds
no arithmetic of the method itself (no quantisation, no permutation, no GEMM): it
only draws the tensors a Mixture-of-Experts layer would receive -- activations,
expert weights, an upstream gradient, and the router's top-k choice -- with the
shapes and distributions of the workloads below.

Router note: the router sits upstream of the expert MLP, so its output (expert ids
and routing probabilities per token) is an *input* here. Probabilities are a softmax
over all experts of N(0,1) logits, the top-k are taken (lowest expert id wins a tie)
and are not renormalised.

Everything is drawn on the CPU with ``torch.Generator().manual_seed(seed)`` in fp32
and then cast, so every consumer sees identical bytes.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int          # tokens
    H: int          # hidden size
    F: int          # expert FFN width (gate and up are each F wide)
    E: int          # experts
    k: int          # top-k
    seed: int
    routing: str = "softmax"   # "softmax" | "dead_last" | "zipf"
    backward: bool = True

    @property
    def M(self) -> int:
        return self.T * self.k

    @property
    def fwd_flops(self) -> float:
        return 6.0 * self.M * self.H * self.F

    @property
    def fwdbwd_flops(self) -> float:
        return 18.0 * self.M * self.H * self.F


CONFIGS = {
    "tiny": MoEConfig("tiny", 1024, 256, 512, 4, 2, seed=1, backward=False),
    "small": MoEConfig("small", 4096, 1024, 2816, 8, 2, seed=2, routing="dead_last"),
    "mixtral": MoEConfig("mixtral", 8192, 4096, 14336, 8, 2, seed=3),
    "mixtral_zipf": MoEConfig("mixtral_zipf", 8192, 4096, 14336, 8, 2, seed=4, routing="zipf"),
    "genomics": MoEConfig("genomics", 32768, 2048, 5632, 64, 8, seed=5),
}

ZIPF_S = 1.2
ZIPF_SMALL_EXPERT_TOKENS = 40
# A large finite logit stands in for "+inf" so that the softmax stays finite.
FORCED_LOGIT = 30.0


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(seed * 1000 + stream)
    return g


def _randn(shape, std, g, dtype=torch.bfloat16, chunk_rows=None):
    """N(0, std^2) in fp32, cast to ``dtype``; drawn in chunks along dim 0 to bound memory."""
    if chunk_rows is None or shape[0] <= chunk_rows:
        return (torch.randn(shape, generator=g) * std).to(dtype)
    out = torch.empty(shape, dtype=dtype)
    for s in range(0, shape[0], chunk_rows):
        e = min(shape[0], s + chunk_rows)
        out[s:e] = (torch.randn((e - s,) + tuple(shape[1:]), generator=g) * std).to(dtype)
    return out


def topk_from_logits(logits: torch.Tensor, k: int):
    """softmax over all experts, then the k largest (ties: lowest index first)."""
    probs = torch.softmax(logits.double(), dim=-1)
    # stable descending order: sort by (-p, index)
    E = logits.shape[-1]
    order = torch.argsort(-probs, dim=-1, stable=True)
    idx = order[:, :k].to(torch.int32)
    p = torch.gather(probs, 1, order[:, :k].long()).to(torch.float32)
    del E
    return idx.contiguous(), p.contiguous()


def _zipf_targets(E: int, s: float = ZIPF_S):
    w = [(e + 1) ** (-s) for e in range(E)]
    tot = sum(w)
    return [x / tot for x in w]


def _zipf_logits(T, E, k, g):
    base = torch.randn((T, E), generator=g)
    forced = torch.randperm(T, generator=g)[:ZIPF_SMALL_EXPERT_TOKENS]
    targets = _zipf_targets(E)
    logw = torch.tensor([math.log(x) for x in targets], dtype=torch.float32)

    def make(beta):
        lg = base + beta * logw
        lg[:, E - 1] = -math.inf
        lg[forced, E - 1] = FORCED_LOGIT
        return lg

    def share0(beta):
        idx, _ = topk_from_logits(make(beta), k)
        return float((idx == 0).sum()) / (T * k)

    lo, hi = 0.0, 20.0
    for _ in range(40):  # deterministic bisection on expert 0's share
        mid = 0.5 * (lo + hi)
        if share0(mid) < targets[0]:
            lo = mid
        else:
            hi = mid
    return make(0.5 * (lo + hi))


def make_routing(cfg: MoEConfig):
    """Router output for ``cfg``: (topk_idx int32[T,k], probs fp32[T,k])."""
    g = _gen(cfg.seed, 1)
    if cfg.routing == "zipf":
        logits = _zipf_logits(cfg.T, cfg.E, cfg.k, g)
    else:
        logits = torch.randn((cfg.T, cfg.E), generator=g)
        if cfg.routing == "dead_last":
            logits[:, cfg.E - 1] = -math.inf
    return topk_from_logits(logits, cfg.k)


def make_activations(cfg: MoEConfig):
    """x bf16[T,H] ~ N(0,1)."""
    return _randn((cfg.T, cfg.H), 1.0, _gen(cfg.seed, 2), chunk_rows=4096)


def make_weights(cfg: MoEConfig):
    """W1 bf16[E,2F,H] (rows 0..F-1 gate, F..2F-1 up) and W2 bf16[E,H,F], both ~N(0,0.02)."""
    W1 = _randn((cfg.E, 2 * cfg.F, cfg.H), 0.02, _gen(cfg.seed, 3), chunk_rows=1)
    W2 = _randn((cfg.E, cfg.H, cfg.F), 0.02, _gen(cfg.seed, 4), chunk_rows=1)
    return W1, W2


def make_grad_output(cfg: MoEConfig):
    """dY bf16[T,H] ~ N(0,1)."""
    return _randn((cfg.T, cfg.H), 1.0, _gen(cfg.seed, 5), chunk_rows=4096)


def make_all(cfg: MoEConfig):
    idx, probs = make_routing(cfg)
    x = make_activations(cfg)
    W1, W2 = make_weights(cfg)
    dy = make_grad_output(cfg) if cfg.backward else None
    return dict(topk_idx=idx, probs=probs, x=x, W1=W1, W2=W2, dy=dy)


def custom(name="custom", T=64, H=128, F=128, E=3, k=2, seed=7, routing="softmax", backward=True):
    return MoEConfig(name, T, H, F, E, k, seed=seed, routing=routing, backward=backward)


def random_matrix(rows, cols, seed, std=1.0, dtype=torch.bfloat16, batch=None):
    """Plain seeded N(0,std^2) matrix (or batch of matrices) for kernel-level tests."""
    g = _gen(seed, 9)
    shape = (rows, cols) if batch is None else (batch, rows, cols)
    return _randn(shape, std, g, dtype=dtype)


def make_expert_weights(cfg: MoEConfig, e: int):
    """Expert e's (W1[e], W2[e]), identical to the slices of make_weights(cfg), drawn
    without materialising the other experts (earlier experts are drawn and dropped)."""
    g1, g2 = _gen(cfg.seed, 3), _gen(cfg.seed, 4)
    w1 = w2 = None
    for i in range(e + 1):
        w1 = (torch.randn((1, 2 * cfg.F, cfg.H), generator=g1) * 0.02).to(torch.bfloat16)
        w2 = (torch.randn((1, cfg.H, cfg.F), generator=g2) * 0.02).to(torch.bfloat16)
    return w1[0], w2[0]


def make_weights_on(cfg: MoEConfig, device):
    """W1 bf16[E,2F,H] and W2 bf16[E,H,F] ~N(0,0.02) drawn on ``device`` with a seeded
    generator of that device, one expert at a time: the full-size workloads hold billions
    of weights, which take minutes to draw on the CPU. Same shapes and distributions as
    make_weights, different values."""
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed * 1000 + 6)
    W1 = torch.empty((cfg.E, 2 * cfg.F, cfg.H), dtype=torch.bfloat16, device=device)
    W2 = torch.empty((cfg.E, cfg.H, cfg.F), dtype=torch.bfloat16, device=device)
    for e in range(cfg.E):
        W1[e] = (torch.randn((2 * cfg.F, cfg.H), generator=g, device=device) * 0.02).to(torch.bfloat16)
        W2[e] = (torch.randn((cfg.H, cfg.F), generator=g, device=device) * 0.02).to(torch.bfloat16)
    return W1, W2
