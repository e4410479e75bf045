"""Seeded synthetic inputs for the Flint MoE layer: activations, router and expert weights.

This module is shared by the CUDA path's tests/bench and by the oracle's; it
holds none of the layer's arithmetic (no quantisation, routing, FFN or combine).
It only draws random numbers and shapes the router so that the logits have the
structure each workload asks for. Random streams are keyed by (seed, purpose,
layer, ...) so any piece can be regenerated on its own.

Generators: numpy's Philox bit generator on the host; torch's CUDA Philox
generator for the multi-gigabyte weight sets that are drawn directly on the GPU.
The two do not produce the same numbers: every comparison copies the arrays one
side used to the other side.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


# ----------------------------------------------------------------- workloads
@dataclass(frozen=True)
class Workload:
    name: str
    d: int
    inter: int
    E: int
    k: int
    S: int
    T: int
    layers: int = 1
    router: str = "plain"       # "plain" | "overlap" | "zipf"
    wdtype: str = "nvfp4"       # "nvfp4" | "bf16"
    residual: bool = False
    std: float = 0.02
    extra: dict = field(default_factory=dict)


# The five layer configurations (shapes the pages leave open are fixed here).
CONFIGS = {
    # reduced layer: d=512, 32 routed + 1 shared, I=128, 4 tokens
    "cfg0": Workload("cfg0", d=512, inter=128, E=32, k=6, S=1, T=4),
    # Flint-shaped layer, decode batch 1
    "cfg1": Workload("cfg1", d=2048, inter=512, E=256, k=6, S=1, T=1),
    # batch 8 with ~40% of each token's experts shared with another token
    "cfg2": Workload("cfg2", d=2048, inter=512, E=256, k=6, S=1, T=8, router="overlap",
                     extra={"p_reuse": 0.27}),
    # 47 stacked layers with a residual between them, batch 1 and 4
    "cfg3_t1": Workload("cfg3_t1", d=2048, inter=512, E=256, k=6, S=1, T=1, layers=47,
                        residual=True),
    "cfg3_t4": Workload("cfg3_t4", d=2048, inter=512, E=256, k=6, S=1, T=4, layers=47,
                        residual=True),
    # batch 64 with a Zipf(1.1) expert-popularity bias, NVFP4 and bf16 weights
    "cfg4_nvfp4": Workload("cfg4_nvfp4", d=2048, inter=512, E=256, k=6, S=1, T=64,
                           router="zipf", extra={"zipf_s": 1.1}),
    "cfg4_bf16": Workload("cfg4_bf16", d=2048, inter=512, E=256, k=6, S=1, T=64,
                          router="zipf", wdtype="bf16", extra={"zipf_s": 1.1}),
}

_PURPOSE = {"x": 1, "router": 2, "experts": 3, "targets": 4, "zipf": 5}


def key(seed: int, purpose: str, *parts: int) -> int:
    ss = np.random.SeedSequence([int(seed), _PURPOSE[purpose]] + [int(p) for p in parts])
    return int(ss.generate_state(1, np.uint64)[0])


def rng(seed: int, purpose: str, *parts: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key(seed, purpose, *parts)))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32/float64 array -> bf16 bit patterns (torch's round-to-nearest-even cast)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------- activations
def x_bits(seed: int, T: int, d: int, stream: int = 0) -> np.ndarray:
    """x ~ N(0, 1), rounded to bf16: uint16 [T][d]."""
    return to_bf16_bits(rng(seed, "x", stream).standard_normal((T, d), dtype=np.float32))


# ----------------------------------------------------------------- expert weights
def expert_weights_np(seed: int, layer: int, expert: int, d: int, inter: int, std: float = 0.02):
    """(gate [I][d], up [I][d], down [d][I]) float32, N(0, std)."""
    g = rng(seed, "experts", layer, expert)
    w = g.standard_normal((3, inter * d), dtype=np.float32) * np.float32(std)
    return w[0].reshape(inter, d), w[1].reshape(inter, d), w[2].reshape(d, inter)


def layer_weights_torch(seed: int, layer: int, n_experts: int, d: int, inter: int,
                        std: float = 0.02, device="cuda"):
    """All experts of one layer drawn at once on `device`: float32 [n][3][I*d]
    (matrix 0 gate [I][d], 1 up [I][d], 2 down [d][I], each flattened)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(key(seed, "experts", layer) & 0x7FFFFFFFFFFFFFFF)
    w = torch.randn((n_experts, 3, inter * d), generator=gen, device=device, dtype=torch.float32)
    return w.mul_(std)


# ----------------------------------------------------------------- router
def router_plain(seed: int, d: int, E: int, layer: int = 0, std: float = 0.02) -> np.ndarray:
    """W_r ~ N(0, std) drawn as d x E, returned transposed as [E][d] float64 (pre-bf16)."""
    w = rng(seed, "router", layer).standard_normal((d, E), dtype=np.float32) * np.float32(std)
    return np.ascontiguousarray(w.T).astype(np.float64)


def _shape_router(w: np.ndarray, x: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """Add a rank-T term D to W_r ([E][d]) with D x_t = bias[t] for every token t
    (least-norm solution through the T x T Gram matrix of the tokens)."""
    gram = x @ x.T                                  # [T][T]
    coef = np.linalg.solve(gram, bias)              # [T][E]
    return w + coef.T @ x                           # [E][d]


def _draw_targets(g, T, E, k, p_reuse):
    sets = []
    used = []
    for t in range(T):
        s = []
        for _ in range(k):
            pool = [e for e in used if e not in s]
            if pool and g.random() < p_reuse:
                e = int(pool[g.integers(len(pool))])
            else:
                free = [e for e in range(E) if e not in used and e not in s]
                e = int(free[g.integers(len(free))])
            s.append(e)
        sets.append(s)
        used.extend(e for e in s if e not in used)
    return sets


def overlap_targets(seed: int, T: int, E: int, k: int, p_reuse: float, target: float = 0.4,
                    tol: float = 0.05):
    """Per token a set of k target experts; each slot reuses, with probability
    p_reuse, an expert already picked by another token, else draws a fresh one.
    Draws are repeated (deterministically, by sub-stream) until the fraction of
    selections shared with another token is within tol of target."""
    sets = None
    for attempt in range(1000):
        sets = _draw_targets(rng(seed, "targets", T, E, k, attempt), T, E, k, p_reuse)
        if T < 2 or abs(overlap_fraction(np.array(sets)) - target) <= tol:
            break
    return sets


def overlap_fraction(ids: np.ndarray) -> float:
    """Fraction of (token, expert) selections whose expert another token also selected."""
    T = ids.shape[0]
    hit = 0
    for t in range(T):
        others = set(ids[np.arange(T) != t].ravel().tolist())
        hit += sum(1 for e in ids[t] if int(e) in others)
    return hit / ids.size


def zipf_bias(seed: int, E: int, s: float) -> np.ndarray:
    """ln p_e with p_e proportional to rank(e)^-s over a seeded permutation of ranks."""
    ranks = rng(seed, "zipf", E).permutation(E) + 1
    p = ranks.astype(np.float64) ** (-s)
    p /= p.sum()
    return np.log(p)


def router_for_targets(w: Workload, seed: int, x_bits_: np.ndarray, sets, boost: float = 8.0,
                       layer: int = 0) -> np.ndarray:
    """Router weights [E][d] as bf16 bits that steer token t to the experts in
    sets[t]: +boost on their logits through a rank-T change of W_r."""
    wr = router_plain(seed, w.d, w.E, layer, w.std)
    x = bf16_bits_to_f64(x_bits_)
    bias = np.zeros((x.shape[0], w.E))
    for t, s in enumerate(sets):
        bias[t, list(s)] = boost
    return to_bf16_bits(_shape_router(wr, x, bias))


def make_router(w: Workload, seed: int, x_bits_: np.ndarray, layer: int = 0) -> np.ndarray:
    """Router weights [E][d] as bf16 bits, shaped for the workload's routing structure."""
    wr = router_plain(seed, w.d, w.E, layer, w.std)
    x = bf16_bits_to_f64(x_bits_)
    if w.router == "overlap":
        # +4 on each token's target experts (logit std is about 0.9 here). A reuse
        # probability of 0.27 gives about 40% overlapping selections at T=8, k=6,
        # E=256 (union of about 38 experts), measured over seeds 0..19.
        sets = overlap_targets(seed + layer, x.shape[0], w.E, w.k, w.extra.get("p_reuse", 0.27))
        bias = np.zeros((x.shape[0], w.E))
        for t, s in enumerate(sets):
            bias[t, s] = 4.0
        wr = _shape_router(wr, x, bias)
    elif w.router == "zipf":
        b = zipf_bias(seed, w.E, w.extra.get("zipf_s", 1.1))
        bias = np.tile(b - b.mean(), (x.shape[0], 1))
        wr = _shape_router(wr, x, bias)
    return to_bf16_bits(wr)
