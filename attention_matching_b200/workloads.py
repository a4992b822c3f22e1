"""Seeded synthetic inputs for KV compaction problems.

This module only draws random numbers and lays them out; it holds none of
the compaction arithmetic, so both the CPU oracle's tests and the CUDA path
consume exactly the same arrays from it.

The pages ("Fast KV Compaction via Attention Matching", the zhichai.net deep
dive §2.2-§2.4 and the xinfinite.net article §5) evaluate on QuALITY,
LongHealth and AIME 2025 with Qwen3-4B / Llama-3.1-8B; neither the datasets
nor the weights are available, so heads shaped like those models stand in:

* ``iid``      - small i.i.d. head: K, Q ~ N(0,1)·d^-1/4, V ~ N(0,1).
* ``structured`` - per head a rank-32 key subspace: K = 2·U·Bᵀ + 0.3·E,
  four large-norm "sink" keys at positions 0-3, reference queries that are
  Dirichlet mixtures of four random keys plus 0.3·noise, V ~ N(0,1).
* ``twin keys`` - a structured head whose every key is followed by a jittered
  copy (repeated tokens); OMP then picks near-duplicate pairs and the NNLS
  refits keep moving weight between them, so variables leave the passive set
  often (a stress case for the refit rather than a page workload).

All draws use ``numpy.random.default_rng(seed)`` (PCG64) in float64 and are
then rounded once to the storage dtype (fp32, or bf16 round-to-nearest-even
through torch's CPU cast).  Every array is returned both as the storage
tensor (what the GPU reads) and as its exact float64 upcast (what the oracle
reads).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

_DT = {"bf16": torch.bfloat16, "fp32": torch.float32}


def round_to(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Round a float64 array once to the storage dtype (RNE), as a CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(_DT[dtype])


def upcast(t: torch.Tensor) -> np.ndarray:
    """Exact float64 view of a stored tensor (bf16 and fp32 embed in fp64)."""
    return t.detach().to("cpu").to(torch.float64).numpy()


@dataclasses.dataclass
class Head:
    """One compaction problem in storage dtype plus its float64 upcast."""
    Q: torch.Tensor          # [n, d]
    K: torch.Tensor          # [T, d]
    V: torch.Tensor          # [T, d]
    key_bias: Optional[np.ndarray] = None   # [T] float32-valued prior bias, or None

    @property
    def n(self) -> int:
        return self.Q.shape[0]

    @property
    def T(self) -> int:
        return self.K.shape[0]

    @property
    def d(self) -> int:
        return self.K.shape[1]

    def f64(self):
        return upcast(self.Q), upcast(self.K), upcast(self.V)


def iid_head(seed: int, n: int, T: int, d: int, dtype: str = "fp32") -> Head:
    """Small i.i.d. head: Q, K ~ N(0,1)·d^-1/4, V ~ N(0,1) (draw order Q, K, V)."""
    rng = np.random.default_rng(seed)
    s = d ** -0.25
    Q = rng.standard_normal((n, d)) * s
    K = rng.standard_normal((T, d)) * s
    V = rng.standard_normal((T, d))
    return Head(round_to(Q, dtype), round_to(K, dtype), round_to(V, dtype))


def _structured_keys(rng: np.random.Generator, T: int, d: int, rank: int,
                     sinks: int, B: np.ndarray) -> np.ndarray:
    U = rng.standard_normal((T, rank))
    E = rng.standard_normal((T, d))
    K = 2.0 * U @ B.T + 0.3 * E
    if sinks:
        med = float(np.median(np.linalg.norm(K, axis=1)))
        for s in range(min(sinks, T)):
            z = rng.standard_normal(rank)
            u = B @ (z / np.linalg.norm(z))
            K[s] = 4.0 * med * u
    return K


def _mixture_queries(rng: np.random.Generator, K: np.ndarray, n: int,
                     first: int = 0) -> np.ndarray:
    """q = Σ_{l<4} a_l k_{j_l} + 0.3·ε with a ~ Dirichlet(1,1,1,1) and the j_l
    uniform over keys [first, T) (sink keys are never mixture components, so
    a query's logit range stays that of an ordinary key match)."""
    T, d = K.shape
    j = rng.integers(first, T, size=(n, 4))
    a = rng.dirichlet(np.ones(4), size=n)
    return np.einsum("nl,nld->nd", a, K[j]) + 0.3 * rng.standard_normal((n, d))


def structured_head(seed: int, n: int, T: int, d: int = 128, rank: int = 32,
                    sinks: int = 4, dtype: str = "bf16", sink_queries: bool = False) -> Head:
    """Structured head (rank-32 keys + noise, sink keys, mixture queries).

    Draw order: basis B (QR of an N(0,1) d×rank matrix), U, E, one unit vector
    per sink, then the query mixture indices, Dirichlet weights and noise,
    then V.  ``sink_queries`` lets the sink keys be mixture components too
    (the mixture indices then range over every key): a query that mixes a
    sink in reaches logits near 130, far above the other queries' best ones.
    """
    rng = np.random.default_rng(seed)
    B, _ = np.linalg.qr(rng.standard_normal((d, rank)))
    K = _structured_keys(rng, T, d, rank, sinks, B)
    Kr = upcast(round_to(K, dtype))
    Q = _mixture_queries(rng, Kr, n, first=0 if sink_queries else min(sinks, T - 1))
    V = rng.standard_normal((T, d))
    return Head(round_to(Q, dtype), round_to(K, dtype), round_to(V, dtype))


def twin_keys_head(seed: int, n: int, T: int, jitter: float = 0.3, d: int = 128,
                   dtype: str = "bf16") -> Head:
    """A structured head of T//2 keys (its own queries and values), each key
    followed by a copy plus jitter·N(0,1) noise with a fresh N(0,1) value:
    keys 2i and 2i+1 are near duplicates.  T must be even."""
    base = structured_head(seed, n=n, T=T // 2, d=d, dtype=dtype)
    rng = np.random.default_rng(seed + 7777)
    K0, V0 = upcast(base.K), upcast(base.V)
    K = np.empty((T, d))
    V = np.empty((T, d))
    K[0::2], V[0::2] = K0, V0
    K[1::2] = K0 + jitter * rng.standard_normal(K0.shape)
    V[1::2] = rng.standard_normal(V0.shape)
    return Head(base.Q.clone(), round_to(K, dtype), round_to(V, dtype))


def long_sequence_chunks(seed: int, T_total: int, chunk: int, n: int, d: int = 128,
                         rank: int = 32, dtype: str = "bf16") -> List[Head]:
    """One long structured key/value sequence split KV-based into contiguous
    chunks (sinks only at global positions 0-3, hence only in chunk 0); each
    chunk gets its own reference queries drawn against its own keys."""
    rng = np.random.default_rng(seed)
    B, _ = np.linalg.qr(rng.standard_normal((d, rank)))
    K = _structured_keys(rng, T_total, d, rank, 4, B)
    V = rng.standard_normal((T_total, d))
    Kt, Vt = round_to(K, dtype), round_to(V, dtype)
    heads = []
    for c0 in range(0, T_total, chunk):
        c1 = min(T_total, c0 + chunk)
        qrng = np.random.default_rng(seed + 100000 * (c0 // chunk + 1))
        Q = _mixture_queries(qrng, upcast(Kt[c0:c1]), n, first=4 if c0 == 0 else 0)
        heads.append(Head(round_to(Q, dtype), Kt[c0:c1].clone(), Vt[c0:c1].clone()))
    return heads


def budget_for_ratio(T: int, ratio: float) -> int:
    """t = round-half-up(T / ratio), at least 1."""
    return max(1, int(math.floor(T / ratio + 0.5)))


def lognormal_budgets(seed: int, num_heads: int, total: int, sigma: float = 0.8,
                      lo: int = 4, hi: int = 1024) -> List[int]:
    """Non-uniform per-head budgets: raw_h = exp(sigma·z_h), a common scale s
    found by bisection so that Σ clip(s·raw_h, lo, hi) = total, then floored
    with the remainder handed out by largest fractional part (ties → lower h)."""
    rng = np.random.default_rng(seed)
    raw = np.exp(sigma * rng.standard_normal(num_heads))

    def tot(s):
        return float(np.clip(s * raw, lo, hi).sum())

    a, b = 0.0, 1.0
    while tot(b) < total:
        b *= 2.0
    for _ in range(200):
        mid = 0.5 * (a + b)
        if tot(mid) < total:
            a = mid
        else:
            b = mid
    x = np.clip(b * raw, lo, hi)
    base = np.floor(x).astype(np.int64)
    rem = int(total - base.sum())
    frac = x - base
    order = sorted(range(num_heads), key=lambda h: (-frac[h], h))
    for h in order:
        if rem <= 0:
            break
        if base[h] < hi:
            base[h] += 1
            rem -= 1
    return [int(v) for v in base]


# ----------------------------------------------------------------------------
# Named workloads (sizes of the pages' settings; see module docstring)
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    name: str
    heads: List[Head]
    budgets: List[int]
    topk: int
    refit_every: int
    dtype: str
    note: str = ""
    key_offsets: Optional[List[int]] = None   # set when the heads' key counts differ


def key_offsets_of(heads: List[Head]) -> List[int]:
    """Row offsets of each head's keys when the heads' K (and V) are stacked
    end to end: [0, T_0, T_0 + T_1, ...]."""
    out = [0]
    for h in heads:
        out.append(out[-1] + h.T)
    return out


def single_head_fp32(seed: int = 1000) -> Workload:
    """One i.i.d. fp32 head, T=256, d=64, n=512, t=16, plain OMP (k=1, R=1)."""
    h = iid_head(seed, n=512, T=256, d=64, dtype="fp32")
    return Workload("single_head_fp32_T256_n512_d64_t16", [h], [16], 1, 1, "fp32")


def qwen3_4b_layer(num_heads: int = 8, T: int = 8192, n: int = 8192, ratio: float = 50.0,
                   seed_base: int = 2000) -> Workload:
    """One Qwen3-4B-shaped layer: 8 KV heads, d=128, T=n=8192, bf16, 50× (t=164),
    top-k=4 with a refit every 2 rounds."""
    heads = [structured_head(seed_base + h, n=n, T=T) for h in range(num_heads)]
    t = budget_for_ratio(T, ratio)
    return Workload(f"qwen3_4b_layer_H{num_heads}_T{T}_n{n}_d128_t{t}", heads,
                    [t] * num_heads, 4, 2, "bf16")


def qwen3_4b_model(num_heads: int = 288, T: int = 8192, n: int = 8192, ratio: float = 50.0,
                   seed_base: int = 4000, only: Optional[List[int]] = None) -> Workload:
    """Full Qwen3-4B-shaped model (36 layers × 8 KV heads) with log-normal
    non-uniform budgets summing to T·H/ratio, clipped to [4, 1024].  ``only``
    keeps the listed heads (their own seeds and budgets), in that order."""
    total = int(math.floor(T * num_heads / ratio + 0.5))
    budgets = lognormal_budgets(seed_base + 999, num_heads, total)
    keep = list(range(num_heads)) if only is None else [int(h) for h in only]
    heads = [structured_head(seed_base + h, n=n, T=T) for h in keep]
    name = f"qwen3_4b_model_H{num_heads}_T{T}_n{n}_d128_lognormal"
    if only is not None:
        name += f"_{len(keep)}of{num_heads}heads"
    return Workload(name, heads, [budgets[h] for h in keep], 4, 2, "bf16")


def llama31_8b_longctx(num_layers: int = 32, kv_heads: int = 8, T_total: int = 60000, chunk: int = 8192,
                       n: int = 8192, ratio: float = 10.0, seed_base: int = 5000,
                       max_sequences: Optional[int] = None) -> Workload:
    """Llama-3.1-8B-shaped long context at 10×: per (layer, KV head) one
    structured sequence of T_total keys cut KV-based into chunks of `chunk`
    keys (the last one shorter: 60000 = 7·8192 + 2656), each chunk with its
    own n reference queries; every chunk is an independent problem with budget
    round-half-up(T_c / ratio) (819 and 266), top-k 8 with a refit every 2
    rounds.  Heads are ordered (layer, KV head, chunk); their key counts
    differ, so the workload carries key offsets.  ``max_sequences`` keeps only
    the first sequences (a smaller sample of the same workload)."""
    seqs = num_layers * kv_heads if max_sequences is None else min(max_sequences, num_layers * kv_heads)
    heads: List[Head] = []
    for q in range(seqs):
        heads.extend(long_sequence_chunks(seed_base + q, T_total, chunk, n))
    budgets = [budget_for_ratio(h.T, ratio) for h in heads]
    name = f"llama31_8b_longctx_{seqs}seq_T{T_total}_chunk{chunk}_n{n}_d128_x{int(ratio)}"
    return Workload(name, heads, budgets, 8, 2, "bf16", key_offsets=key_offsets_of(heads))


# ----------------------------------------------------------------------------
# Online compaction rounds (xinfinite.net article §5 and Table 3: a fixed
# physical cache; everything but the latest tokens is compacted by half,
# repeatedly).  Each head keeps its rank-32 key basis across rounds; a round's
# cache is [previous compacted keys (their β as prior key bias)] + [kept
# latest tokens] + [fresh tokens], and reference queries are drawn against
# the whole current cache.  The compacted values enter the next round rounded
# to the storage dtype, as a cache would hold them.
# ----------------------------------------------------------------------------

class OnlineHeads:
    def __init__(self, num_heads: int, cache: int = 2048, keep: int = 20, n: int = 2048, d: int = 128,
                 rank: int = 32, seed: int = 3000, dtype: str = "bf16"):
        self.H, self.cache, self.keep, self.n, self.d, self.rank = num_heads, cache, keep, n, d, rank
        self.dtype = dtype
        self.round = 0
        self.rngs = [np.random.default_rng(seed + h) for h in range(num_heads)]
        self.bases = [np.linalg.qr(r.standard_normal((d, rank)))[0] for r in self.rngs]
        self.prev = None     # per head: (K f64, V f64, bias f64) of the uncompacted tail + compacted block

    @property
    def compact_len(self) -> int:
        return self.cache - self.keep

    @property
    def budget(self) -> int:
        return budget_for_ratio(self.compact_len, 2.0)

    def _fresh(self, h: int, count: int, sinks: int):
        rng = self.rngs[h]
        K = _structured_keys(rng, count, self.d, self.rank, sinks, self.bases[h])
        V = rng.standard_normal((count, self.d))
        return upcast(round_to(K, self.dtype)), upcast(round_to(V, self.dtype))

    def next_round(self, compacted=None) -> List[Head]:
        """Heads of the next round.  `compacted` (after the first round) is a
        per-head list of (C_k, beta, C_v) from the previous round's output."""
        heads = []
        for h in range(self.H):
            if self.round == 0:
                K, V = self._fresh(h, self.cache, sinks=4)
                bias = np.zeros(self.cache)
            else:
                Ck, beta, Cv = compacted[h]
                Kp, Vp, _ = self.prev[h]
                kept_K, kept_V = Kp[self.compact_len:], Vp[self.compact_len:]
                nf = self.cache - len(Ck) - self.keep
                Kf, Vf = self._fresh(h, nf, sinks=0)
                K = np.vstack([np.asarray(Ck, np.float64), kept_K, Kf])
                V = np.vstack([upcast(round_to(np.asarray(Cv, np.float64), self.dtype)), kept_V, Vf])
                bias = np.concatenate([np.asarray(beta, np.float64), np.zeros(self.keep + nf)])
            # the four sink keys lead the cache in the first round and, being
            # selected first, lead every compacted block after it
            Q = _mixture_queries(self.rngs[h], K, self.n, first=4)
            self.prev = (self.prev or [None] * self.H)
            self.prev[h] = (K, V, bias)
            c = self.compact_len
            heads.append(Head(round_to(Q, self.dtype), round_to(K[:c], self.dtype), round_to(V[:c], self.dtype),
                              key_bias=np.float32(bias[:c])))
        self.round += 1
        return heads


def sensitivity_curves(seed: int, num_heads: int, levels: int, t_min: int = 4, quantum: int = 16,
                       convex: bool = True) -> np.ndarray:
    """Synthetic per-head sensitivity curves [num_heads][levels]: head h's loss
    at budget t = t_min + g·quantum is a_h·exp(−(t − t_min)/τ_h) + c_h, with
    a_h = exp(N(0, 1)), τ_h = 64·exp(0.7·N(0, 1)) and c_h ~ U(0, 0.1):
    decreasing with diminishing returns, heads differing in scale and in how
    fast they saturate (the pages' curves need models and data).  With
    convex=False each head also gets a bump of height 0.3·a_h at a random
    level, so that some gains grow before they shrink."""
    rng = np.random.default_rng(seed)
    a = np.exp(rng.standard_normal(num_heads))
    tau = 64.0 * np.exp(0.7 * rng.standard_normal(num_heads))
    c = rng.uniform(0.0, 0.1, num_heads)
    t = t_min + quantum * np.arange(levels, dtype=np.float64)
    L = a[:, None] * np.exp(-(t[None, :] - t_min) / tau[:, None]) + c[:, None]
    if not convex:
        at = rng.integers(0, levels, num_heads)
        L[np.arange(num_heads), at] += 0.3 * a
    return L
