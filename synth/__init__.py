"""Seeded synthetic workloads for the MAC-Attention decode step.

This module only draws inputs: query streams, KV caches, block tables and
sequence lengths.  It holds none of the method's arithmetic (no RoPE, no
distances, no softmax, no merge), so both the fp64 oracle and the CUDA path
can consume its output without sharing any computation.

Shapes follow the workloads of the MAC-Attention page (page 1, abstract):
long-context decode with GQA, contiguous or paged bf16 KV, a short window of
recent queries, and a mix of "near-repeat" queries (which the match stage is
meant to hit) and fresh ones.  The public benchmark suites named there are
not available; these synthetic streams take their shapes instead.

Recipe (all draws from numpy PCG64 streams keyed by (seed, tag, chunk)):
  * K, V ~ N(0, 1), drawn in float32 and rounded once to bf16 (round to
    nearest even); the bf16 bit patterns are what both sides read.
  * Query stream, step by step, sequence by sequence: a step labelled "hit"
    copies the pre-RoPE query of one uniformly chosen step among the last W
    steps of the same sequence (all Hq heads together) and adds N(0, sigma^2)
    per element; a "fresh" step draws N(0, 1).  A hit label on a step whose
    window is still empty falls back to fresh.
  * Labels: iid Bernoulli, a per-sequence Bernoulli rate, or a two-state
    Markov chain, depending on the workload.
  * With head_labels, the label and the source step are drawn per query head
    (each head repeats its own earlier query or draws fresh on its own), so
    the heads of one KV head's group disagree; otherwise all Hq heads of a
    sequence share them.
The distance margins that keep match decisions away from ties are a property
of these distributions (sigma small against 1); the tests check them with the
oracle rather than here.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor
from typing import Optional, Tuple

import numpy as np

# Stream tags for independent PCG64 streams.
_TAG_K = 1
_TAG_V = 2
_TAG_Q = 3
_TAG_LAYOUT = 4

_CHUNK_ELEMS = 1 << 22  # elements per independently seeded KV chunk


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode workload.

    Attributes follow the MAC-Attention page's notation where it has one:
    W is the match window, band the amend band b, tau the match threshold.
    """
    name: str
    B: int                 # sequences in the batch
    Hq: int                # query heads
    Hkv: int               # KV heads (GQA group G = Hq // Hkv)
    D: int                 # head dim
    L0: Tuple[int, ...]    # context length of each sequence before decode step 0
    steps: int             # decode steps in the stream
    W: int                 # match window (recent queries)
    band: int              # amend band b (keys recomputed before the match)
    tau: float             # match threshold on the mean squared L2 distance
    sigma: float           # std of the perturbation added to a repeated query
    rope_theta: float
    page_size: int         # 0 = contiguous KV, else tokens per page
    hit_model: Tuple       # ("iid", p) | ("per_seq", lo, hi) | ("markov", stay_hit, stay_miss)
    seed: int
    append: bool = False   # the step's own K/V row arrives through an append call
    head_labels: bool = False  # repeat labels and sources drawn per query head

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def seq_lens(self, t: int) -> np.ndarray:
        """Keys visible at decode step t (the step's own row included)."""
        return np.asarray([l0 + t + 1 for l0 in self.L0], dtype=np.int32)

    def capacity(self, steps: Optional[int] = None) -> int:
        """Largest sequence length reached over `steps` decode steps."""
        steps = self.steps if steps is None else steps
        return max(self.L0) + steps


def _tau(d: int, sigma: float) -> float:
    # Threshold of the tiny workload's definition, 0.5 * d * sigma^2 * 4,
    # applied to every workload (the larger ones state sigma but not tau).
    return 0.5 * d * sigma * sigma * 4.0


def _paged_L0(seed: int, B: int, lo: int, hi: int) -> Tuple[int, ...]:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(_TAG_LAYOUT, 0))))
    return tuple(int(x) for x in rng.integers(lo, hi + 1, size=B))


WORKLOADS = {
    "tiny": Workload(
        name="tiny", B=1, Hq=4, Hkv=1, D=64, L0=(1024,), steps=64, W=16, band=32,
        tau=_tau(64, 0.01), sigma=0.01, rope_theta=1e4, page_size=0,
        hit_model=("iid", 0.5), seed=0),
    "llama8b_32k": Workload(
        name="llama8b_32k", B=1, Hq=32, Hkv=8, D=128, L0=(32768,), steps=256, W=32, band=256,
        tau=_tau(128, 0.02), sigma=0.02, rope_theta=5e5, page_size=0,
        hit_model=("iid", 0.7), seed=1),
    "long_128k": Workload(
        name="long_128k", B=4, Hq=32, Hkv=8, D=128, L0=(131072,) * 4, steps=128, W=32, band=256,
        tau=_tau(128, 0.02), sigma=0.02, rope_theta=5e5, page_size=0,
        hit_model=("iid", 0.9), seed=2),
    "paged_mixed": Workload(
        name="paged_mixed", B=16, Hq=32, Hkv=8, D=128, L0=_paged_L0(3, 16, 8192, 65536), steps=64,
        W=32, band=128, tau=_tau(128, 0.02), sigma=0.02, rope_theta=5e5, page_size=16,
        hit_model=("per_seq", 0.3, 0.95), seed=3),
    "continuous_16k": Workload(
        name="continuous_16k", B=8, Hq=32, Hkv=8, D=128, L0=(16384,) * 8, steps=4096, W=64, band=256,
        tau=_tau(128, 0.02), sigma=0.02, rope_theta=5e5, page_size=16,
        hit_model=("markov", 0.9, 0.5), seed=4, append=True),
}


def all_miss(wl: Workload) -> Workload:
    """The same inputs with threshold 0: every step is a miss (dense decode)."""
    return wl.with_(name=wl.name + "_allmiss", tau=0.0)


# ----------------------------------------------------------------------------
# query stream
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class QueryStream:
    q: np.ndarray        # [T, B, Hq, D] float32, pre-RoPE
    label: np.ndarray    # [T, B] bool ([T, B, Hq] with head_labels): drawn as a repeat
    src: np.ndarray      # [T, B] int ([T, B, Hq] with head_labels): step index it repeats, -1 if fresh
    rope_pos: np.ndarray  # [T, B] int32, position of the step's token
    seq_lens: np.ndarray  # [T, B] int32, keys visible at the step


def queries(wl: Workload, steps: Optional[int] = None, sigma: Optional[float] = None) -> QueryStream:
    """Draw the pre-RoPE query stream of a workload (deterministic in wl.seed)."""
    T = wl.steps if steps is None else steps
    sig = wl.sigma if sigma is None else sigma
    if wl.head_labels:
        return _queries_per_head(wl, T, sig)
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(wl.seed, spawn_key=(_TAG_Q, 0))))
    B, Hq, D, W = wl.B, wl.Hq, wl.D, wl.W
    q = np.empty((T, B, Hq, D), dtype=np.float32)
    label = np.zeros((T, B), dtype=bool)
    src = np.full((T, B), -1, dtype=np.int64)
    kind = wl.hit_model[0]
    rate = None
    if kind == "per_seq":
        rate = rng.uniform(wl.hit_model[1], wl.hit_model[2], size=B)
    prev_hit = np.zeros(B, dtype=bool)
    for t in range(T):
        for b in range(B):
            u = rng.random()
            if kind == "iid":
                want = u < wl.hit_model[1]
            elif kind == "per_seq":
                want = u < rate[b]
            elif kind == "markov":
                stay_hit, stay_miss = wl.hit_model[1], wl.hit_model[2]
                want = (u < stay_hit) if prev_hit[b] else (u >= stay_miss)
            else:
                raise ValueError(kind)
            occupied = min(t, W)
            if want and occupied > 0:
                s = t - 1 - int(rng.integers(0, occupied))
                noise = rng.standard_normal((Hq, D))
                q[t, b] = (q[s, b].astype(np.float64) + sig * noise).astype(np.float32)
                label[t, b] = True
                src[t, b] = s
            else:
                q[t, b] = rng.standard_normal((Hq, D)).astype(np.float32)
            prev_hit[b] = label[t, b] if kind == "markov" else prev_hit[b]
    lens = np.stack([wl.seq_lens(t) for t in range(T)]) if T else np.zeros((0, B), np.int32)
    return QueryStream(q=q, label=label, src=src, rope_pos=(lens - 1).astype(np.int32), seq_lens=lens)


def _queries_per_head(wl: Workload, T: int, sig: float) -> QueryStream:
    """Query stream whose repeat labels and sources are drawn per query head."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(wl.seed, spawn_key=(_TAG_Q, 1))))
    B, Hq, D, W = wl.B, wl.Hq, wl.D, wl.W
    q = np.empty((T, B, Hq, D), dtype=np.float32)
    label = np.zeros((T, B, Hq), dtype=bool)
    src = np.full((T, B, Hq), -1, dtype=np.int64)
    kind = wl.hit_model[0]
    rate = rng.uniform(wl.hit_model[1], wl.hit_model[2], size=B) if kind == "per_seq" else None
    prev_hit = np.zeros((B, Hq), dtype=bool)
    for t in range(T):
        for b in range(B):
            for h in range(Hq):
                u = rng.random()
                if kind == "iid":
                    want = u < wl.hit_model[1]
                elif kind == "per_seq":
                    want = u < rate[b]
                elif kind == "markov":
                    want = (u < wl.hit_model[1]) if prev_hit[b, h] else (u >= wl.hit_model[2])
                else:
                    raise ValueError(kind)
                occupied = min(t, W)
                if want and occupied > 0:
                    s = t - 1 - int(rng.integers(0, occupied))
                    noise = rng.standard_normal(D)
                    q[t, b, h] = (q[s, b, h].astype(np.float64) + sig * noise).astype(np.float32)
                    label[t, b, h] = True
                    src[t, b, h] = s
                else:
                    q[t, b, h] = rng.standard_normal(D).astype(np.float32)
                prev_hit[b, h] = label[t, b, h]
    lens = np.stack([wl.seq_lens(t) for t in range(T)]) if T else np.zeros((0, B), np.int32)
    return QueryStream(q=q, label=label, src=src, rope_pos=(lens - 1).astype(np.int32), seq_lens=lens)


# ----------------------------------------------------------------------------
# KV cache
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + r) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _fill_normal_bf16(out: np.ndarray, seed: int, tag: int, threads: int = 0) -> None:
    flat = out.reshape(-1)
    n = flat.size
    nchunk = (n + _CHUNK_ELEMS - 1) // _CHUNK_ELEMS

    def work(c: int) -> None:
        lo = c * _CHUNK_ELEMS
        hi = min(n, lo + _CHUNK_ELEMS)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(tag, c))))
        flat[lo:hi] = f32_to_bf16_bits(g.standard_normal(hi - lo, dtype=np.float32))

    if nchunk <= 1:
        for c in range(nchunk):
            work(c)
        return
    import os
    nt = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(nt) as ex:
        list(ex.map(work, range(nchunk)))


@dataclasses.dataclass
class KVCache:
    K: np.ndarray                     # uint16 bf16 bits: [B, max_seq, Hkv, D] or [P, page, Hkv, D]
    V: np.ndarray
    block_table: Optional[np.ndarray]  # [B, max_pages_per_seq] int32 (-1 = unused) or None
    max_seq: int                      # per-sequence capacity (contiguous) / pages*page (paged)
    num_pages: int                    # 0 for contiguous

    @property
    def paged(self) -> bool:
        return self.block_table is not None


def kv_cache(wl: Workload, steps: Optional[int] = None) -> KVCache:
    """Draw the KV cache holding every row the stream will read.

    Contiguous: rows [0, L0 + steps) of every sequence.  Paged: each sequence
    owns ceil((L0_b + steps) / page) pages, assigned from a shared pool by a
    random permutation.
    """
    bt, max_seq, P = kv_layout(wl, steps)
    shape = (wl.B, max_seq, wl.Hkv, wl.D) if bt is None else (P, wl.page_size, wl.Hkv, wl.D)
    K = np.empty(shape, np.uint16)
    V = np.empty(shape, np.uint16)
    _fill_normal_bf16(K, wl.seed, _TAG_K)
    _fill_normal_bf16(V, wl.seed, _TAG_V)
    return KVCache(K, V, bt, max_seq, P)


def kv_layout(wl: Workload, steps: Optional[int] = None):
    """The cache's layout alone: (block_table or None, per-sequence capacity,
    pages in the pool (0 when contiguous)), as kv_cache lays it out."""
    T = wl.steps if steps is None else steps
    cap = wl.capacity(T)
    if wl.page_size == 0:
        return None, cap, 0
    ps = wl.page_size
    npages = [-(-(l0 + T) // ps) for l0 in wl.L0]
    P = int(sum(npages))
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(wl.seed, spawn_key=(_TAG_LAYOUT, 1))))
    perm = rng.permutation(P).astype(np.int32)
    maxp = max(npages)
    bt = np.full((wl.B, maxp), -1, np.int32)
    off = 0
    for b, n in enumerate(npages):
        bt[b, :n] = perm[off:off + n]
        off += n
    return bt, maxp * ps, P


def kv_row(cache: KVCache, b: int, pos: int) -> Tuple[np.ndarray, np.ndarray]:
    """The [Hkv, D] K and V rows of sequence b at position pos (bf16 bits)."""
    if not cache.paged:
        return cache.K[b, pos], cache.V[b, pos]
    ps = cache.K.shape[1]
    page = cache.block_table[b, pos // ps]
    return cache.K[page, pos % ps], cache.V[page, pos % ps]


def step_rows(cache: KVCache, seq_lens: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """[B, Hkv, D] rows at position seq_lens-1 of every sequence (the step's own token)."""
    ks, vs = zip(*(kv_row(cache, b, int(L) - 1) for b, L in enumerate(seq_lens)))
    return np.stack(ks), np.stack(vs)


def dense_equiv_kv_bytes(wl: Workload, seq_lens: np.ndarray) -> int:
    """bf16 K+V bytes a dense decode of this step reads (all keys of every unit)."""
    return int(np.sum(seq_lens.astype(np.int64))) * wl.Hkv * wl.D * 2 * 2
