"""Seeded synthetic inputs for the deterministic MoE layer.

This module only draws random numbers and names workload shapes. It holds
none of the layer's arithmetic (no top-k, no softmax, no schedule, no FFN),
so that the CPU oracle and the CUDA path can both be fed from it without
sharing any computation.

Workloads (shapes follow the Kimi-2.5 case study in "Mixture-of-Kittens: A MoE
Megakernel for GB300 NVL72", section 3 "The Goldilocks Minibatch Size T", and
the scheduler benchmark in "Scan once, scatter once", section "Measured,
including where it loses"):

  tiny   P=1 x 512 tokens,  H=256,  I=128,  E=8,   top-2
  sched  P=8 x 7168 tokens, E=384, top-8, expert ids only (uniform, no repeats)
  mid    P=4 x 4096 tokens, H=2048, I=1024, E=64,  top-4
  kimi   P=8 x 7168 tokens, H=7168, I=2048, E=384, top-8 (transfer slice 2368)
  zipf   kimi shapes, expert choice ~ Zipf(1.2) over a seeded expert
         permutation, plus 8 experts that are never chosen
  tiny_bwd  P=2 x 256 tokens, H=256, I=256, E=8, top-2 (small backward case)

Distributions: router logits fp32 N(0,1); activations bf16 N(0,1); SwiGLU
weights W1, W3 [E,H,I] and W2 [E,I,H] bf16 N(0, 0.02). Seeds are
1000 * workload_id + stream_id.
"""
from __future__ import annotations

import dataclasses
import random

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    wid: int          # workload id, used for seeds
    P: int            # logical expert-parallel peers
    N: int            # tokens per peer
    E: int            # experts
    k: int            # routes per token
    H: int = 0        # hidden size (0 = scheduler-only workload)
    I: int = 0        # expert intermediate size
    pad: int = 256    # expert segment padding in rows
    logits: str = "normal"   # "normal" | "zipf" | "ids" (scheduler-only)
    n_empty: int = 0         # experts forced never to be chosen
    minibatch: int = 0       # transfer slice T in tokens per peer (0 = all)

    @property
    def n_tokens(self) -> int:
        return self.P * self.N

    @property
    def n_routes(self) -> int:
        return self.P * self.N * self.k

    def shape(self) -> dict:
        return dict(P=self.P, N=self.N, E=self.E, k=self.k, H=self.H, I=self.I, pad=self.pad)


WORKLOADS = {
    "tiny": Workload("tiny", 0, P=1, N=512, E=8, k=2, H=256, I=128),
    "sched": Workload("sched", 1, P=8, N=7168, E=384, k=8, logits="ids"),
    "mid": Workload("mid", 2, P=4, N=4096, E=64, k=4, H=2048, I=1024),
    "kimi": Workload("kimi", 3, P=8, N=7168, E=384, k=8, H=7168, I=2048, minibatch=2368),
    "zipf": Workload("zipf", 4, P=8, N=7168, E=384, k=8, H=7168, I=2048, logits="zipf", n_empty=8),
    # Kimi expert shapes with 16 experts and ~1,200 routes each (as at full size):
    # a few GB on the device, for profiler captures of the FFN kernels
    "kimi_e16": Workload("kimi_e16", 5, P=1, N=2400, E=16, k=8, H=7168, I=2048),
    # smallest backward case: the backward's GEMMs need I % 256 == 0
    "tiny_bwd": Workload("tiny_bwd", 6, P=2, N=256, E=8, k=2, H=256, I=256),
}


def seed_for(wid: int, stream_id: int) -> int:
    return 1000 * wid + stream_id


# stream ids
_S_LOGITS, _S_X, _S_W1, _S_W3, _S_W2, _S_PERM, _S_EMPTY, _S_IDS, _S_Y, _S_DOUT = range(10)


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_logits(w: Workload) -> torch.Tensor:
    """Router logits fp32 [P*N, E] on the CPU."""
    T, E = w.n_tokens, w.E
    if w.logits == "normal":
        out = torch.randn((T, E), generator=_gen(seed_for(w.wid, _S_LOGITS)), dtype=torch.float32)
    elif w.logits == "zipf":
        # Gumbel-top-k over log-weights -1.2*ln(rank) draws k distinct experts
        # per token with Zipf(1.2) probabilities (sampling without replacement).
        perm = torch.randperm(E, generator=_gen(seed_for(w.wid, _S_PERM)))
        rank = torch.empty(E, dtype=torch.float64)
        rank[perm] = torch.arange(1, E + 1, dtype=torch.float64)
        base = (-1.2 * torch.log(rank)).to(torch.float32)
        u = torch.rand((T, E), generator=_gen(seed_for(w.wid, _S_LOGITS)), dtype=torch.float32)
        u = u.clamp_(min=1e-12, max=1.0 - 1e-7)
        out = base.unsqueeze(0) - torch.log(-torch.log(u))
    else:
        raise ValueError(f"workload {w.name} has no router logits")
    if w.n_empty:
        g = _gen(seed_for(w.wid, _S_EMPTY))
        empty = torch.randperm(E, generator=g)[: w.n_empty]
        out[:, empty] = float("-inf")
    return out.contiguous()


def empty_experts(w: Workload) -> list[int]:
    """Experts forced to -inf logits (never chosen) in workload w."""
    if not w.n_empty:
        return []
    g = _gen(seed_for(w.wid, _S_EMPTY))
    return sorted(torch.randperm(w.E, generator=g)[: w.n_empty].tolist())


def make_ids_uniform(P: int, N: int, E: int, k: int, seed: int) -> torch.Tensor:
    """Expert ids int32 [P, N, k]: per token, k distinct experts uniformly at random."""
    if P * N == 0:
        return torch.zeros((P, N, k), dtype=torch.int32)
    g = _gen(seed)
    keys = torch.rand((P * N, E), generator=g)
    ids = torch.argsort(keys, dim=1)[:, :k].to(torch.int32)
    return ids.reshape(P, N, k).contiguous()


def make_sched_ids(w: Workload) -> torch.Tensor:
    return make_ids_uniform(w.P, w.N, w.E, w.k, seed_for(w.wid, _S_IDS))


def make_x(w: Workload, device="cpu") -> torch.Tensor:
    """Token activations bf16 [P*N, H]."""
    g = _gen(seed_for(w.wid, _S_X), device)
    return torch.randn((w.n_tokens, w.H), generator=g, dtype=torch.bfloat16, device=device)


def make_expert_outputs(w: Workload, rows: int, device="cpu") -> torch.Tensor:
    """Stand-in expert output rows fp32 [rows, H] ~ N(0, 0.05^2) (about the spread
    of real expert outputs at these weight scales), for checking the combine
    stage on inputs that neither side computed."""
    g = _gen(seed_for(w.wid, _S_Y), device)
    t = torch.randn((rows, w.H), generator=g, dtype=torch.float32, device=device)
    return t.mul_(0.05)


def make_dout(w: Workload, device="cpu") -> torch.Tensor:
    """Upstream gradient of the layer output, bf16 [P*N, H] ~ N(0,1)."""
    g = _gen(seed_for(w.wid, _S_DOUT), device)
    return torch.randn((w.n_tokens, w.H), generator=g, dtype=torch.bfloat16, device=device)


def make_weights(w: Workload, device="cpu"):
    """SwiGLU expert weights (W1 gate, W3 up [E,H,I]; W2 down [E,I,H]), bf16 N(0, 0.02).

    Drawn with torch's generator on `device`; the same seed gives different
    (but equally distributed) values on the CPU and on the GPU, so every test
    hands the very same tensors to both sides.
    """
    out = []
    for sid, shp in ((_S_W1, (w.E, w.H, w.I)), (_S_W3, (w.E, w.H, w.I)), (_S_W2, (w.E, w.I, w.H))):
        g = _gen(seed_for(w.wid, sid), device)
        t = torch.randn(shp, generator=g, dtype=torch.bfloat16, device=device)
        t.mul_(0.02)
        out.append(t)
    return tuple(out)


def sweep_cases(n_cases: int = 945, seed: int = 945, max_P: int = 8, max_E: int = 64,
                max_N: int = 512, max_k: int = 8):
    """Randomised small scheduler cases: P in 1..8, E in 1..64, N in 1..512, k in 1..min(8,E).

    Mirrors the randomized validation set of "Scan once, scatter once"
    (section "The fix is a counting sort"). Yields (P, N, E, k, ids[P,N,k]).
    """
    rng = random.Random(seed)
    for c in range(n_cases):
        P = rng.randint(1, max_P)
        E = rng.randint(1, max_E)
        N = rng.randint(1, max_N)
        k = rng.randint(1, min(max_k, E))
        pattern = rng.random()
        if pattern < 0.70:
            ids = make_ids_uniform(P, N, E, k, seed * 100000 + c)
        else:
            # adversarial: a few hot experts take most routes
            g = _gen(seed * 100000 + c)
            hot = max(1, E // 8)
            keys = torch.rand((P * N, E), generator=g)
            keys[:, :hot] += 1.0
            ids = torch.argsort(keys, dim=1, descending=True)[:, :k].to(torch.int32)
            perm = torch.randperm(E, generator=g).to(torch.int32)
            ids = perm[ids.long()].reshape(P, N, k).contiguous()
        yield P, N, E, k, ids


def sample_tokens(n_tokens: int, n: int, seed: int) -> list[int]:
    """n distinct token indices in [0, n_tokens), sorted, always including the first and last."""
    rng = random.Random(seed)
    n = min(n, n_tokens)
    picks = set([0, n_tokens - 1]) if n_tokens else set()
    while len(picks) < n:
        picks.add(rng.randrange(n_tokens))
    return sorted(picks)


__all__ = [
    "Workload", "WORKLOADS", "seed_for", "make_logits", "make_ids_uniform", "make_sched_ids",
    "make_x", "make_weights", "make_expert_outputs", "make_dout", "sweep_cases",
    "sample_tokens", "empty_experts",
]
