"""Seeded synthetic inputs for the ROSA retrieval step.

This module only draws random inputs (numpy PCG64, and torch generators for
the large bf16 tensors).  It holds none of the retrieval arithmetic, so both
the CUDA path and the CPU oracle can be fed from it.

Five workloads, each with its seed, follow the shapes of the ROSA-Tuning
setting (arXiv 2602.02499: section 3.2 multi-route symbol streams, section
4.1 parallelism over batch x route, section 5.1 M = 4 on Qwen3-1.7B):

1. ``binary-4k``       1 stream, T=4096, K=2, i.i.d. Bernoulli(0.5), q = k.
2. ``planted-16``      4 x 32 streams, T=16384, K=16 uniform with planted
                       copy segments (length 32..256) whose disjoint
                       destinations cover 5% of each stream (a later copy may
                       overwrite an earlier one's source), q = k.
3. ``qwen-proj-64``    B=1, T=32768: bf16 hidden states N(0,1) of width 2048,
                       seeded Gaussian projections W_q, W_k (N(0, 1/2048)) to
                       64 channels; M=1 gives 64 binary routes; value rows
                       V ~ N(0,1) with d=128 per route.
4. ``zipf-256-131k``   128 streams, T=131072, K=256 Zipf(s=1.1) symbols,
                       query and key drawn independently but sharing planted
                       exact repeats (length 16..1024) covering >= 2% of the
                       query positions.
5. ``markov-4-train``  B=8 x 256 streams, T=8192, K=4 Markov chain (stay 0.7,
                       otherwise uniform over the other 3 symbols), query and
                       key independent; value rows d=64 per route.

Every generator takes size overrides so that tests can draw the same recipe
at a size the CPU oracle finishes in seconds.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

LAG_DEFAULT = 2


@dataclass
class SymbolWorkload:
    name: str
    B: int
    R: int
    T: int
    K: int
    g: int
    q: np.ndarray            # uint8 [S, T]
    k: np.ndarray            # uint8 [S, T]; the same object as q when q = k
    seed: int
    notes: dict = field(default_factory=dict)

    @property
    def S(self) -> int:
        return self.B * self.R

    @property
    def same_qk(self) -> bool:
        return self.q is self.k


def _zipf_p(K: int, s: float) -> np.ndarray:
    r = np.arange(1, K + 1, dtype=np.float64)
    p = r ** (-s)
    return p / p.sum()


def binary_iid(T: int = 4096, S: int = 1, seed: int = 1, g: int = LAG_DEFAULT) -> SymbolWorkload:
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 2, size=(S, T), dtype=np.uint8)
    return SymbolWorkload("binary-4k", 1, S, T, 2, g, q, q, seed)


def planted_copies(B: int = 4, R: int = 32, T: int = 16384, K: int = 16, seed: int = 2,
                   cover: float = 0.05, lmin: int = 32, lmax: int = 256,
                   g: int = LAG_DEFAULT) -> SymbolWorkload:
    """Uniform symbols with copy segments of the stream's own earlier content.

    Repeat until ``cover`` of the positions lie in a destination: length
    l ~ U[lmin, lmax]; destination start d uniform with destinations kept
    disjoint; source start uniform in [0, d - l]; copy k[src:src+l] to d.
    """
    rng = np.random.default_rng(seed)
    S = B * R
    k = rng.integers(0, K, size=(S, T), dtype=np.uint8)
    lmax = min(lmax, max(lmin, T // 4))
    for s in range(S):
        taken = np.zeros(T, dtype=bool)
        covered = 0
        tries = 0
        while covered < cover * T and tries < 10000:
            tries += 1
            ell = int(rng.integers(lmin, lmax + 1))
            if 2 * ell > T:
                break
            d = int(rng.integers(ell, T - ell + 1))
            if taken[d:d + ell].any():
                continue
            src = int(rng.integers(0, d - ell + 1))
            k[s, d:d + ell] = k[s, src:src + ell]
            taken[d:d + ell] = True
            covered += ell
    return SymbolWorkload("planted-16", B, R, T, K, g, k, k, seed)


def zipf_planted(S: int = 128, T: int = 131072, K: int = 256, zipf_s: float = 1.1,
                 seed_q: int = 41, seed_k: int = 42, seed_plant: int = 43,
                 cover: float = 0.02, lmin: int = 16, lmax: int = 1024,
                 g: int = LAG_DEFAULT) -> SymbolWorkload:
    """Independent Zipf query/key streams sharing planted exact repeats.

    Repeat until ``cover`` of the query positions are planted: a payload of
    length l ~ U[lmin, lmax] drawn from the same Zipf law is written at key
    position a and at query position b >= a + l + g, key and query plants
    each kept disjoint.
    """
    p = _zipf_p(K, zipf_s)
    rq = np.random.default_rng(seed_q)
    rk = np.random.default_rng(seed_k)
    rp = np.random.default_rng(seed_plant)
    q = rq.choice(K, size=(S, T), p=p).astype(np.uint8)
    k = rk.choice(K, size=(S, T), p=p).astype(np.uint8)
    lmax = min(lmax, max(lmin, T // 4))
    for s in range(S):
        tk = np.zeros(T, dtype=bool)
        tq = np.zeros(T, dtype=bool)
        covered = 0
        tries = 0
        while covered < cover * T and tries < 10000:
            tries += 1
            ell = int(rp.integers(lmin, lmax + 1))
            if 2 * ell + g > T:
                break
            a = int(rp.integers(0, T - 2 * ell - g + 1))
            b = int(rp.integers(a + ell + g, T - ell + 1))
            if tk[a:a + ell].any() or tq[b:b + ell].any():
                continue
            payload = rp.choice(K, size=ell, p=p).astype(np.uint8)
            k[s, a:a + ell] = payload
            q[s, b:b + ell] = payload
            tk[a:a + ell] = True
            tq[b:b + ell] = True
            covered += ell
    return SymbolWorkload("zipf-256-131k", 1, S, T, K, g, q, k, seed_q)


def markov(B: int = 8, R: int = 256, T: int = 8192, K: int = 4, stay: float = 0.7,
           seed_q: int = 51, seed_k: int = 52, g: int = LAG_DEFAULT) -> SymbolWorkload:
    """Markov-chain symbols: keep the previous symbol with probability ``stay``,
    otherwise move to one of the other K-1 symbols uniformly; uniform start."""
    S = B * R

    def chain(seed):
        rng = np.random.default_rng(seed)
        start = rng.integers(0, K, size=(S, 1))
        move = rng.random((S, T - 1)) >= stay
        step = rng.integers(1, K, size=(S, T - 1)) * move
        inc = np.concatenate([start, step], axis=1)
        return (np.cumsum(inc, axis=1) % K).astype(np.uint8)

    return SymbolWorkload("markov-4-train", B, R, T, K, g, chain(seed_q), chain(seed_k), seed_q)


# --------------------------------------------------------------------------
# bf16 tensors (torch; drawn on the given device with a seeded generator)
# --------------------------------------------------------------------------

def bf16_normal(shape, seed: int, device="cpu", std: float = 1.0):
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def qwen_projection_inputs(T: int = 32768, width: int = 2048, channels: int = 64, B: int = 1,
                           seed_h: int = 3, seed_wq: int = 31, seed_wk: int = 32, device="cpu"):
    """Hidden states H [B, T, width] ~ N(0,1) and projections W_q, W_k
    [width, channels] ~ N(0, 1/width), all bf16.  The caller forms
    q_vec = H @ W_q and k_vec = H @ W_k (set-up, outside the retrieval step)."""
    H = bf16_normal((B, T, width), seed_h, device)
    Wq = bf16_normal((width, channels), seed_wq, device, std=width ** -0.5)
    Wk = bf16_normal((width, channels), seed_wk, device, std=width ** -0.5)
    return H, Wq, Wk


def value_rows(B: int, T: int, width: int, seed: int, device="cpu"):
    """Value rows V [B, T, width] ~ N(0,1) bf16."""
    return bf16_normal((B, T, width), seed, device)


# --------------------------------------------------------------------------
# registry of the five full-size workloads
# --------------------------------------------------------------------------

WORKLOADS = {
    1: dict(name="binary-4k", kind="symbols", make=lambda: binary_iid()),
    2: dict(name="planted-16", kind="symbols", make=lambda: planted_copies()),
    3: dict(name="qwen-proj-64", kind="hidden", T=32768, width=2048, channels=64, M=1,
            d=128, rho=128, seed_v=33),
    4: dict(name="zipf-256-131k", kind="symbols", make=lambda: zipf_planted()),
    5: dict(name="markov-4-train", kind="symbols", make=lambda: markov(), d=64, rho=64, seed_v=53),
}


def spec(name: str) -> dict:
    """The registry entry of the workload called ``name``."""
    for v in WORKLOADS.values():
        if v["name"] == name:
            return v
    raise KeyError(name)
