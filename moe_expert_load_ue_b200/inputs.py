"""Seeded synthetic inputs for the balancer's hot path.

This module only draws inputs: post-gating top-k expert ids (and, for the
small case, their softmax gates), expert weights and replica gradients.  It
holds none of the balancer's arithmetic (no histogram, plan, reroute, copy or
reduction), so that the CUDA path and the CPU oracle can both consume the same
inputs without sharing any of the method's code.

Routing model.  The UltraEP pages (arXiv 2606.04101, news summary "Comment
fonctionne l'équilibrage en 300 microsecondes") describe production routing
that is skewed and non-stationary.  We stand in for those traces with a Zipf
popularity over a seeded permutation of experts, p_e ∝ (pi(e) + 1)^-s, and
draw each token's K distinct experts by Gumbel-top-k on log p_e (highest
perturbed score first, so position k = 0 is the token's top choice).  Tokens
are drawn in fixed chunks of 16384 with their own child seeds, so the ids do
not depend on how many threads generate them.  The
106B/671B workloads re-draw the permutation every microbatch (non-stationary
load); the extreme-skew workload additionally forces one hot expert into 30 %
of the tokens.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Iterator

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: routing shape, EP layout and expert shapes.

    E experts, top-K, N simulated EP ranks with H = E / N home slots and R
    redundant slots each, ``tokens_per_rank`` tokens per rank (T = N * that),
    Zipf exponent ``s``.  Expert weights are 3 bf16 matrices rows x cols (P =
    3 * rows * cols elements); replica gradients are fp32 or bf16.
    """

    name: str
    E: int
    K: int
    N: int
    R: int
    tokens_per_rank: int
    s: float
    microbatches: int = 1
    repermute: bool = True          # re-draw the popularity permutation per microbatch
    rows: int = 1024
    cols: int = 512
    grad_dtype: str = "fp32"        # "fp32" or "bf16"
    hot_fraction: float = 0.0       # share of tokens forced onto one hot expert
    base_seed: int = 0

    @property
    def H(self) -> int:
        return self.E // self.N

    @property
    def T(self) -> int:
        return self.N * self.tokens_per_rank

    @property
    def L(self) -> int:
        return self.T * self.K

    @property
    def S(self) -> int:
        return self.N * (self.H + self.R)

    @property
    def P(self) -> int:
        return 3 * self.rows * self.cols

    def seed(self, microbatch: int) -> int:
        return self.base_seed * 1000 + microbatch

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workload families of the balancer's evaluation, at their stated sizes.
TINY = Workload("tiny", E=64, K=8, N=8, R=2, tokens_per_rank=512, s=1.0,
                microbatches=1, repermute=False, rows=1024, cols=512, grad_dtype="fp32")
CLASS_106B = Workload("106B-class", E=128, K=8, N=32, R=2, tokens_per_rank=8192, s=1.2,
                      microbatches=16, rows=4096, cols=1408, grad_dtype="fp32")
CLASS_671B = Workload("671B-class", E=256, K=8, N=64, R=1, tokens_per_rank=4096, s=1.2,
                      microbatches=16, rows=7168, cols=2048, grad_dtype="bf16")
EXTREME = Workload("extreme-skew", E=256, K=8, N=256, R=1, tokens_per_rank=1024, s=1.6,
                   microbatches=16, rows=2048, cols=1024, grad_dtype="fp32", hot_fraction=0.3)

WORKLOADS = {w.name: w for w in (TINY, CLASS_106B, CLASS_671B, EXTREME)}


def sweep(seeds: int = 5) -> Iterator[Workload]:
    """The sweep grid: E=256, top-8, one redundant slot per rank (E + N slots)."""
    for tpr in (256, 1024, 4096, 16384, 32768):
        for n in (8, 32, 64, 128, 256):
            for s in (0.0, 0.8, 1.2, 1.6):
                for seed in range(seeds):
                    yield Workload(f"sweep-tpr{tpr}-n{n}-s{s}-seed{seed}", E=256, K=8, N=n, R=1,
                                   tokens_per_rank=tpr, s=s, microbatches=1,
                                   rows=2048, cols=1024, grad_dtype="fp32", base_seed=seed)


def zipf_popularity(E: int, s: float, rng: np.random.Generator) -> np.ndarray:
    """p_e ∝ (pi(e) + 1)^-s over a seeded permutation pi of the experts (float64)."""
    perm = rng.permutation(E)
    p = (perm.astype(np.float64) + 1.0) ** (-s)
    return p / p.sum()


_CHUNK = 16384            # tokens per independently seeded chunk (fixed: keeps draws thread-count independent)


def _topk_chunk(seed_seq: np.random.SeedSequence, n: int, inv_p: np.ndarray, K: int) -> np.ndarray:
    """Gumbel-top-k for n tokens.  With G = -log(X), X ~ Exp(1), G is standard
    Gumbel noise, and log p_e + G_e orders the experts exactly as X_e / p_e
    does in reverse, so the K smallest X_e / p_e are the K largest perturbed
    scores, in the same order (the exponential-race form of Gumbel-top-k)."""
    rng = np.random.default_rng(seed_seq)
    E = inv_p.shape[0]
    x = rng.standard_exponential((n, E), dtype=np.float32)
    x *= inv_p
    if K < E:
        part = np.argpartition(x, K - 1, axis=1)[:, :K]
    else:
        part = np.tile(np.arange(E), (n, 1))
    sc = np.take_along_axis(x, part, axis=1)
    order = np.argsort(sc, axis=1, kind="stable")
    return np.take_along_axis(part, order, axis=1).astype(np.int32)


def _gumbel_topk(p: np.ndarray, T: int, K: int, seed_seq: np.random.SeedSequence) -> np.ndarray:
    """K distinct experts per token, ordered by decreasing perturbed score."""
    with np.errstate(divide="ignore"):
        inv_p = (1.0 / p).astype(np.float32)        # p_e = 0 -> never drawn
    n_chunks = (T + _CHUNK - 1) // _CHUNK
    kids = seed_seq.spawn(n_chunks)
    sizes = [min(_CHUNK, T - i * _CHUNK) for i in range(n_chunks)]
    out = np.empty((T, K), dtype=np.int32)
    if n_chunks == 0:
        return out
    workers = max(1, min(8, os.cpu_count() or 1, n_chunks))
    with ThreadPoolExecutor(workers) as ex:
        parts = list(ex.map(lambda a: _topk_chunk(kids[a], sizes[a], inv_p, K), range(n_chunks)))
    for i, part in enumerate(parts):
        out[i * _CHUNK:i * _CHUNK + sizes[i]] = part
    return out


def popularity(w: Workload, microbatch: int = 0) -> np.ndarray:
    """Expert popularity p_e of a microbatch (re-permuted per microbatch unless stationary)."""
    mb = microbatch if w.repermute else 0
    ss_perm = np.random.SeedSequence(w.seed(mb)).spawn(3)[0]
    return zipf_popularity(w.E, w.s, np.random.default_rng(ss_perm))


def topk_ids(w: Workload, microbatch: int = 0) -> np.ndarray:
    """Post-gating top-K expert ids, int32 [T, K], row-major (token-major)."""
    _, ss_hot, ss_draw = np.random.SeedSequence(w.seed(microbatch)).spawn(3)
    p = popularity(w, microbatch)
    if w.hot_fraction <= 0.0:
        return _gumbel_topk(p, w.T, w.K, ss_draw)
    # One hot expert forced into floor(hot_fraction * T) tokens as their top
    # choice; every other draw excludes it so its count is exact.
    rng_hot = np.random.default_rng(ss_hot)
    hot = int(rng_hot.integers(w.E))
    n_hot = int(math.floor(w.hot_fraction * w.T))
    hot_tokens = rng_hot.choice(w.T, size=n_hot, replace=False)
    p_x = p.copy()
    p_x[hot] = 0.0
    ids = _gumbel_topk(p_x, w.T, w.K, ss_draw)
    ids[hot_tokens, 1:] = ids[hot_tokens, :-1]
    ids[hot_tokens, 0] = hot
    return ids


def topk_ids_device(w: Workload, microbatch: int = 0, device="cuda"):
    """Same routing model drawn with torch on `device` (for large sweeps; a
    different random stream from topk_ids).  Returns int32 [T, K] on device."""
    import torch
    p = torch.as_tensor(popularity(w, microbatch), dtype=torch.float32, device=device)
    g = torch.Generator(device=device).manual_seed(w.seed(microbatch) * 7919 + 17)
    out = torch.empty((w.T, w.K), dtype=torch.int32, device=device)
    inv = 1.0 / p
    chunk = 1 << 16
    for a in range(0, w.T, chunk):
        b = min(w.T, a + chunk)
        x = torch.empty((b - a, w.E), dtype=torch.float32, device=device).exponential_(generator=g)
        x *= inv                       # exponential race: the K smallest X / p are the Gumbel-top-k
        out[a:b] = torch.topk(x, w.K, dim=1, largest=False, sorted=True).indices.to(torch.int32)
    return out


def hot_expert(w: Workload, microbatch: int = 0) -> int:
    """The forced hot expert of an extreme-skew microbatch (same draw as topk_ids)."""
    ss_hot = np.random.SeedSequence(w.seed(microbatch)).spawn(3)[1]
    return int(np.random.default_rng(ss_hot).integers(w.E))


def gates(ids: np.ndarray, w: Workload, microbatch: int = 0) -> np.ndarray:
    """fp32 softmax gates over each token's K chosen experts (carried along by the dispatch layout)."""
    rng = np.random.default_rng(w.seed(microbatch) + 7_000_000)
    logits = rng.standard_normal(ids.shape).astype(np.float32)
    logits = -np.sort(-logits, axis=1)
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def random_bf16_bits(shape, std: float, seed: int) -> np.ndarray:
    """Normal(0, std) values rounded to bf16, returned as uint16 bit patterns."""
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(shape, dtype=np.float32) * np.float32(std)).view(np.uint32)
    # round to nearest even on the upper 16 bits
    x = x + (np.uint32(0x7FFF) + ((x >> np.uint32(16)) & np.uint32(1)))
    return (x >> np.uint32(16)).astype(np.uint16)


def random_f32(shape, std: float, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(std)
