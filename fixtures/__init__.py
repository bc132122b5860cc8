"""Seeded synthetic inputs for the routed top-k MoE layer.

This module only *draws* inputs: codebook grids in compact form, packed expert
blocks made of uniform random fields, activations, expert ids and router
weights.  It holds none of the layer's arithmetic (no dequantisation, no
projection, no SiLU, no accumulation), so both the CPU oracle and the CUDA
library can be fed from it without sharing any computation.

Random source: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014).  Output i of a stream is
mix64(state0 + (i + 1) * GAMMA), which makes the generator counter based and
lets numpy draw whole arrays at once.  Each purpose (grid, one matrix of one
expert, x, routing, ...) gets its own stream derived from (seed, tag), so a
subset of experts can be generated without drawing the others.

Packed block layouts follow the layer's two weight formats (IQ2_XS-style,
74 bytes per 256 weights; IQ1_M-style, 56 bytes per 256 weights); the field
offsets are the only format knowledge here and are needed to place the block
scale `d` inside otherwise uniform random bytes.
"""

from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

QTYPE_IQ2XS = 1
QTYPE_IQ1M = 2

BLOCK_WEIGHTS = 256
BLOCK_BYTES = {QTYPE_IQ2XS: 74, QTYPE_IQ1M: 56}
GRID_ENTRIES = {QTYPE_IQ2XS: 512, QTYPE_IQ1M: 2048}
# fp16 exponent fields of the block scale d: IQ2 d in [2^-12, 2^-10), IQ1 d in [2^-9, 2^-7).
_D_EXP_FIELD = {QTYPE_IQ2XS: 3, QTYPE_IQ1M: 6}

SEED_BASE = 0x5EED0000


def _mix64(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def _scalar_mix(v: int) -> int:
    return int(_mix64(np.array([v & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))[0])


def _tag(*parts: int) -> int:
    h = 0x243F6A8885A308D3
    for p in parts:
        h = _scalar_mix(h ^ (int(p) & 0xFFFFFFFFFFFFFFFF))
    return h


class Stream:
    """One SplitMix64 stream, identified by a seed and a tuple of tag integers."""

    def __init__(self, seed: int, *tag: int):
        self.state0 = np.uint64(_scalar_mix(int(seed) ^ _tag(*tag)))
        self.pos = 0

    def u64(self, n: int) -> np.ndarray:
        idx = np.arange(self.pos + 1, self.pos + n + 1, dtype=np.uint64)
        self.pos += n
        with np.errstate(over="ignore"):
            return _mix64(self.state0 + idx * GAMMA)

    def bytes(self, n: int) -> np.ndarray:
        words = self.u64((n + 7) // 8)
        return words.view(np.uint8)[:n].copy()

    def uniform(self, n: int) -> np.ndarray:
        """Doubles in [0, 1)."""
        return (self.u64(n) >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)

    def uniform_open(self, n: int) -> np.ndarray:
        """Doubles in (0, 1]."""
        return ((self.u64(n) >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)

    def randint(self, n: int, hi: int) -> np.ndarray:
        return np.minimum((self.uniform(n) * hi).astype(np.int64), hi - 1)

    def normal(self, n: int) -> np.ndarray:
        """N(0,1) in double by Box-Muller (cosine branch only)."""
        u1 = self.uniform_open(n)
        u2 = self.uniform(n)
        return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


# --------------------------------------------------------------------------- grids


def compact_from_symbols(symbols: np.ndarray) -> np.ndarray:
    """Pack rows of 8 symbols (0..2) into compact uint16 entries, symbol j at bits 2j..2j+1."""
    symbols = np.asarray(symbols, dtype=np.uint32)
    out = np.zeros(symbols.shape[0], dtype=np.uint32)
    for j in range(8):
        out |= symbols[:, j] << np.uint32(2 * j)
    return out.astype(np.uint16)


def make_grid(seed: int, qtype: int) -> np.ndarray:
    """A seeded grid of distinct entries drawn uniformly from the 3^8 symbol patterns."""
    n = GRID_ENTRIES[qtype]
    st = Stream(seed, 1, qtype)
    chosen: List[int] = []
    seen = set()
    while len(chosen) < n:
        for v in st.randint(4 * n, 6561):
            v = int(v)
            if v not in seen:
                seen.add(v)
                chosen.append(v)
                if len(chosen) == n:
                    break
    pats = np.array(chosen, dtype=np.int64)
    syms = np.zeros((n, 8), dtype=np.uint32)
    for j in range(8):
        syms[:, j] = pats % 3
        pats //= 3
    return compact_from_symbols(syms)


# --------------------------------------------------------------------------- packed matrices


def matrix_bytes(qtype: int, rows: int, k: int) -> int:
    n = rows * k
    if n % BLOCK_WEIGHTS:
        raise ValueError("rows*k must be a multiple of 256")
    return (n // BLOCK_WEIGHTS) * BLOCK_BYTES[qtype]


def make_matrix(seed: int, qtype: int, rows: int, k: int, *tag: int) -> np.ndarray:
    """Packed bytes of one matrix: uniform random fields, block scale d a random fp16 in range."""
    nbytes = matrix_bytes(qtype, rows, k)
    nblk = nbytes // BLOCK_BYTES[qtype]
    st = Stream(seed, 2, qtype, rows, k, *tag)
    raw = st.bytes(nbytes).reshape(nblk, BLOCK_BYTES[qtype])
    bits = st.u64(nblk)
    mant = (bits & np.uint64(0x3FF)).astype(np.uint16)
    expo = (np.uint16(_D_EXP_FIELD[qtype]) + ((bits >> np.uint64(10)) & np.uint64(1)).astype(np.uint16))
    d = (expo << np.uint16(10)) | mant
    raw[:, 0] = (d & 0xFF).astype(np.uint8)
    raw[:, 1] = (d >> 8).astype(np.uint8)
    return raw.reshape(-1)


@dataclasses.dataclass
class Expert:
    qtype: int
    ffn: int
    gate: np.ndarray  # packed, F rows x H
    up: np.ndarray  # packed, F rows x H
    down: np.ndarray  # packed, H rows x F

    @property
    def nbytes(self) -> int:
        return self.gate.size + self.up.size + self.down.size


def make_expert(seed: int, qtype: int, hidden: int, ffn: int, expert_id: int) -> Expert:
    return Expert(
        qtype,
        ffn,
        make_matrix(seed, qtype, ffn, hidden, expert_id, 0),
        make_matrix(seed, qtype, ffn, hidden, expert_id, 1),
        make_matrix(seed, qtype, hidden, ffn, expert_id, 2),
    )


def expert_bytes(qtype: int, hidden: int, ffn: int) -> int:
    return 2 * matrix_bytes(qtype, ffn, hidden) + matrix_bytes(qtype, hidden, ffn)


# --------------------------------------------------------------------------- activations / routing


def make_x(seed: int, n_tokens: int, hidden: int, tag: int = 0) -> np.ndarray:
    st = Stream(seed, 3, tag)
    return st.normal(n_tokens * hidden).astype(np.float32).reshape(n_tokens, hidden)


def draw_distinct_nonadjacent(st: Stream, k: int, n_experts: int, exclude=()) -> List[int]:
    """k distinct ids, no two adjacent (|a-b| != 1), avoiding `exclude`."""
    chosen: List[int] = []
    banned = set(exclude)
    while len(chosen) < k:
        for v in st.randint(64, n_experts):
            v = int(v)
            if v in banned or v in chosen or (v - 1) in chosen or (v + 1) in chosen:
                continue
            chosen.append(v)
            if len(chosen) == k:
                break
    return chosen


def normalised_positive_weights(st: Stream, k: int) -> np.ndarray:
    w = 0.5 + st.uniform(k)
    return (w / w.sum()).astype(np.float32)


def softmax_topk_routing(logits: np.ndarray, k: int):
    """Input recipe for the batched-decode workload: softmax over the experts, the k
    largest probabilities (ties to the lower id), renormalised over those k."""
    t, e = logits.shape
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    order = np.lexsort((np.broadcast_to(np.arange(e), (t, e)), -p), axis=1)[:, :k]
    sel = np.take_along_axis(p, order, axis=1)
    w = sel / sel.sum(axis=1, keepdims=True)
    return order.astype(np.int32), w.astype(np.float32)


def zipf_topk_routing(st: Stream, n_tokens: int, n_experts: int, k: int, s: float):
    """Per token k distinct experts drawn Zipf(s) over ranks 1..E (duplicates redrawn),
    rank -> id by a seeded permutation; weights = softmax of N(0,1) logits over the k."""
    ranks = np.arange(1, n_experts + 1, dtype=np.float64)
    pmf = ranks ** (-s)
    cdf = np.cumsum(pmf / pmf.sum())
    cdf[-1] = 1.0
    perm = np.argsort(st.uniform(n_experts), kind="stable")
    ids = np.zeros((n_tokens, k), dtype=np.int32)
    for t in range(n_tokens):
        got: List[int] = []
        while len(got) < k:
            for u in st.uniform(4 * k):
                r = int(np.searchsorted(cdf, u, side="right"))
                r = min(r, n_experts - 1)
                e = int(perm[r])
                if e not in got:
                    got.append(e)
                    if len(got) == k:
                        break
        ids[t] = got
    logits = st.normal(n_tokens * k).reshape(n_tokens, k)
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    w = (p / p.sum(axis=1, keepdims=True)).astype(np.float32)
    return ids, w


# --------------------------------------------------------------------------- the five workloads


@dataclasses.dataclass
class Workload:
    name: str
    seed: int
    hidden: int
    n_experts: int
    ffn: int
    top_k: int
    n_tokens: int
    qtypes: np.ndarray  # [n_experts] int32
    shared_qtype: Optional[int]
    shared_ffn: int
    grid_iq2: np.ndarray
    grid_iq1: np.ndarray
    x: np.ndarray  # [T, H] float32
    ids: np.ndarray  # [T, k] int32
    weights: np.ndarray  # [T, k] float32
    _experts: dict = dataclasses.field(default_factory=dict)

    def expert(self, e: int) -> Expert:
        if e not in self._experts:
            self._experts[e] = make_expert(self.seed, int(self.qtypes[e]), self.hidden, self.ffn, e)
        return self._experts[e]

    def shared(self) -> Optional[Expert]:
        if self.shared_qtype is None:
            return None
        if "shared" not in self._experts:
            self._experts["shared"] = make_expert(self.seed, self.shared_qtype, self.hidden, self.shared_ffn, 1_000_000)
        return self._experts["shared"]

    def selected(self) -> List[int]:
        return sorted(set(int(v) for v in self.ids.reshape(-1)))

    def unique_bytes(self) -> int:
        b = sum(self.expert(e).nbytes for e in self.selected())
        s = self.shared()
        return b + (s.nbytes if s is not None else 0)


WORKLOAD_NAMES = {
    1: "tiny-iq2xs-h256-e16-f64-top4-t1",
    2: "decode-iq2xs-h2048-e512-f512-top10-t1",
    3: "decode-iq1m-cold-h2048-e512-f512-top10-t1",
    4: "batched-decode-mixed-h2048-e512-f512-top10-t64-shared512",
    5: "prefill-iq1m-zipf1.1-h2048-e512-f512-top10-t4096-shared512",
}


def workload(cfg: int, seed: Optional[int] = None, n_tokens: Optional[int] = None) -> Workload:
    """The synthetic inputs of workload `cfg` (1..5).  `n_tokens` shrinks the token
    count of configs 4 and 5 for quick tests (routing is drawn for the first tokens only)."""
    seed = SEED_BASE + cfg if seed is None else seed
    g2 = make_grid(seed, QTYPE_IQ2XS)
    g1 = make_grid(seed, QTYPE_IQ1M)
    if cfg == 1:
        H, E, F, k, T = 256, 16, 64, 4, 1
        qt = np.full(E, QTYPE_IQ2XS, np.int32)
        st = Stream(seed, 4)
        ids = np.array([sorted(int(v) for v in np.argsort(st.uniform(E))[:k])], np.int32)
        w = normalised_positive_weights(st, k)[None, :]
        return Workload(WORKLOAD_NAMES[1], seed, H, E, F, k, T, qt, None, 0, g2, g1, make_x(seed, T, H), ids, w)
    if cfg in (2, 3):
        H, E, F, k, T = 2048, 512, 512, 10, 1
        q = QTYPE_IQ2XS if cfg == 2 else QTYPE_IQ1M
        qt = np.full(E, q, np.int32)
        st = Stream(seed, 4)
        ids = np.array([draw_distinct_nonadjacent(st, k, E)], np.int32)
        w = normalised_positive_weights(st, k)[None, :]
        return Workload(WORKLOAD_NAMES[cfg], seed, H, E, F, k, T, qt, None, 0, g2, g1, make_x(seed, T, H), ids, w)
    if cfg == 4:
        H, E, F, k = 2048, 512, 512, 10
        T = 64 if n_tokens is None else n_tokens
        qt = np.where(np.arange(E) % 2 == 0, QTYPE_IQ2XS, QTYPE_IQ1M).astype(np.int32)
        st = Stream(seed, 4)
        logits = st.normal(64 * E).reshape(64, E)[:T]
        ids, w = softmax_topk_routing(logits, k)
        return Workload(WORKLOAD_NAMES[4], seed, H, E, F, k, T, qt, QTYPE_IQ2XS, 512, g2, g1, make_x(seed, T, H), ids, w)
    if cfg == 5:
        H, E, F, k = 2048, 512, 512, 10
        T = 4096 if n_tokens is None else n_tokens
        qt = np.full(E, QTYPE_IQ1M, np.int32)
        st = Stream(seed, 4)
        ids, w = zipf_topk_routing(st, T, E, k, 1.1)
        return Workload(WORKLOAD_NAMES[5], seed, H, E, F, k, T, qt, QTYPE_IQ1M, 512, g2, g1, make_x(seed, T, H), ids, w)
    raise ValueError(f"unknown workload {cfg}")


def decode_id_sets(seed: int, n_sets: int, k: int, n_experts: int) -> np.ndarray:
    """`n_sets` pairwise-disjoint sets of k distinct, non-adjacent expert ids (so a run
    over all sets touches n_sets*k different experts)."""
    st = Stream(seed, 5)
    used: List[int] = []
    out = np.zeros((n_sets, k), np.int32)
    for s in range(n_sets):
        ids = draw_distinct_nonadjacent(st, k, n_experts, exclude=used)
        used.extend(ids)
        out[s] = ids
    return out


# --------------------------------------------------------------------------- projection formats

PROJ_BLOCK = {3: (32, 34), 4: (256, 144)}  # qtype -> (weights, bytes) per block: Q8_0-style, Q4_K-style


def make_proj_matrix(seed: int, qtype: int, rows: int, k: int, *tag: int) -> np.ndarray:
    """Packed bytes of a Q8_0-style (3) or Q4_K-style (4) matrix: uniform random
    fields, fp16 scales drawn so that |W| stays near 1/sqrt(k) (the scale
    fields are the only format knowledge here: Q8_0 d at bytes 0-1; Q4_K d and
    dmin at bytes 0-1 and 2-3)."""
    bw, bb = PROJ_BLOCK[qtype]
    nblk = rows * k // bw
    st = Stream(seed, 9, qtype, rows, k, *tag)
    raw = st.bytes(nblk * bb).reshape(nblk, bb)
    bits = st.u64(nblk)
    mant = (bits & np.uint64(0x3FF)).astype(np.uint16)
    if qtype == 3:  # d in [2^-13, 2^-12): |w| <= 128 d
        d = (np.uint16(2) << np.uint16(10)) | mant
        raw[:, 0], raw[:, 1] = (d & 0xFF).astype(np.uint8), (d >> 8).astype(np.uint8)
    else:  # d in [2^-12, 2^-11), dmin in [2^-13, 2^-12): |w| <= 63 * 15 d
        d = (np.uint16(3) << np.uint16(10)) | mant
        dm = (np.uint16(2) << np.uint16(10)) | ((bits >> np.uint64(10)) & np.uint64(0x3FF)).astype(np.uint16)
        raw[:, 0], raw[:, 1] = (d & 0xFF).astype(np.uint8), (d >> 8).astype(np.uint8)
        raw[:, 2], raw[:, 3] = (dm & 0xFF).astype(np.uint8), (dm >> 8).astype(np.uint8)
    return raw.reshape(-1)
