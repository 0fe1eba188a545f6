"""Seeded synthetic inputs for NSA selected-block attention.

This module is shared by the oracle tests, the CUDA parity tests and the
benchmark.  It only draws random numbers and builds the block-index input; it
holds none of the attention arithmetic.

Workload recipe (the shapes named on the "Flash-Sparse-Attention" project page,
quick-start section: block_size 64, topk 16, init_blocks 1, local_blocks 2,
varlen lengths [65536, 32768] packed through cu_seqlens):

* Q, K, V, dO: i.i.d. N(0, 1) float32 drawn from ``PCG64(seed)`` in that order,
  then rounded to the nearest bfloat16 (ties to even).  Arrays are returned as
  float32 holding exactly those bfloat16 values.
* block_idx[t, g, :] for token t (local position i, query block qb = i // bs) and
  KV head g: the structural blocks [0, qb, qb - 1] (deduplicated, clipped to
  >= 0), then distinct uniform draws from {1, ..., qb - 2} until ``topk`` entries
  or that range is exhausted, then -1 padding.  Draws come from
  ``PCG64(seed + 1_000_003)``, independently per (token, KV head), with Floyd's
  sampling-without-replacement algorithm.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

INDEX_SEED_OFFSET = 1_000_003


def bf16_round(x: np.ndarray, inplace: bool = False) -> np.ndarray:
    """Round finite float32 values to the nearest bfloat16 (ties to even); return float32.

    On the uint32 bit patterns: add 0x7FFF plus the lowest kept bit, then clear the
    16 dropped bits.  Chunked, so that large arrays need no big temporaries.
    """
    if inplace and isinstance(x, np.ndarray) and x.dtype == np.float32 and x.flags.c_contiguous:
        out = x
    else:
        out = np.array(x, dtype=np.float32, copy=True, order="C")
    bits = out.reshape(-1).view(np.uint32)
    chunk = 1 << 22
    lsb = np.empty(min(chunk, bits.size), dtype=np.uint32)
    for a in range(0, bits.size, chunk):
        seg = bits[a:a + chunk]
        t = lsb[:seg.size]
        np.right_shift(seg, 16, out=t)
        t &= np.uint32(1)
        seg += np.uint32(0x7FFF)
        seg += t
        seg &= np.uint32(0xFFFF0000)
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are already bfloat16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def cu_seqlens_from_lengths(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def _floyd_sample(rng: np.random.Generator, n: np.ndarray, m: np.ndarray, mmax: int) -> np.ndarray:
    """Per row r, m[r] distinct values from {0..n[r]-1} (Floyd's algorithm).

    Returns int64 [rows, mmax]; positions >= m[r] hold -1.  Rows with m[r] > n[r]
    must not be passed (callers clip m to n).
    """
    rows = n.shape[0]
    out = np.full((rows, mmax), -1, dtype=np.int64)
    for it in range(mmax):
        active = it < m
        # j runs over n - m, ..., n - 1
        j = n - m + it
        hi = np.where(active, j + 1, 1)
        t = rng.integers(0, hi)
        if it > 0:
            dup = (out[:, :it] == t[:, None]).any(axis=1)
        else:
            dup = np.zeros(rows, dtype=bool)
        pick = np.where(dup, j, t)
        out[:, it] = np.where(active, pick, -1)
    return out


def make_block_idx(cu_seqlens: np.ndarray, hkv: int, topk: int, block_size: int,
                   seed: int) -> np.ndarray:
    """block_idx int32 [T, hkv, topk] by the rule in the module docstring."""
    rng = np.random.Generator(np.random.PCG64(seed + INDEX_SEED_OFFSET))
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T = int(cu[-1])
    out = np.full((T, hkv, topk), -1, dtype=np.int32)
    for s in range(len(cu) - 1):
        c0, c1 = int(cu[s]), int(cu[s + 1])
        L = c1 - c0
        if L == 0:
            continue
        i = np.arange(L, dtype=np.int64)
        qb = i // block_size
        # structural blocks, in the order [0, qb, qb-1], deduplicated
        st = np.full((L, 3), -1, dtype=np.int64)
        st[:, 0] = 0
        st[:, 1] = np.where(qb >= 1, qb, -1)
        st[:, 2] = np.where(qb >= 2, qb - 1, -1)
        nstruct = 1 + (qb >= 1).astype(np.int64) + (qb >= 2).astype(np.int64)
        nrand_cap = np.maximum(qb - 2, 0)
        nrand = np.clip(topk - nstruct, 0, None)
        nrand = np.minimum(nrand, nrand_cap)
        mmax = max(0, min(topk, int(nrand.max()) if L else 0))
        rows = np.repeat(np.arange(L), hkv)
        n_r = np.repeat(nrand_cap, hkv)
        m_r = np.repeat(nrand, hkv)
        draws = _floyd_sample(rng, n_r, m_r, mmax) if mmax > 0 else np.zeros((L * hkv, 0), np.int64)
        draws = np.where(draws >= 0, draws + 1, -1)          # values in {1..qb-2}
        block = np.full((L * hkv, topk), -1, dtype=np.int64)
        ns = min(3, topk)
        block[:, :ns] = st[rows, :ns]
        # compact structural part (drop the -1 holes; holes only occur at the end)
        nst = np.minimum(np.repeat(nstruct, hkv), topk)
        if mmax > 0:
            col = nst[:, None] + np.arange(mmax)[None, :]
            ok = (np.arange(mmax)[None, :] < m_r[:, None]) & (col < topk)
            rr, cc = np.nonzero(ok)
            block[rr, col[rr, cc]] = draws[rr, cc]
        out[c0:c1] = block.reshape(L, hkv, topk).astype(np.int32)
    return out


def band_block_idx(cu_seqlens: np.ndarray, hkv: int, topk: int, block_size: int,
                   window: int) -> np.ndarray:
    """block_idx int32 [T, hkv, topk] of the sliding branch: for the token at local
    position i (query block qb), the blocks qb, qb - 1, .., down to the block of key
    i - window + 1 (at most ceil(window / block_size) + 1 blocks, never below 0), then
    -1 pads; the same row for every KV head.  No random draws."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T = int(cu[-1])
    nwb = (window + block_size - 1) // block_size + 1
    if nwb > topk:
        raise ValueError("topk is smaller than the number of blocks a window reaches")
    out = np.full((T, hkv, topk), -1, dtype=np.int32)
    for s in range(len(cu) - 1):
        c0, c1 = int(cu[s]), int(cu[s + 1])
        qb = np.arange(c1 - c0, dtype=np.int64) // block_size
        blocks = qb[:, None] - np.arange(nwb, dtype=np.int64)[None, :]
        out[c0:c1, :, :nwb] = np.where(blocks >= 0, blocks, -1)[:, None, :].astype(np.int32)
    return out


@dataclasses.dataclass
class Problem:
    """One synthetic problem.  Float arrays are float32 holding bf16 values."""
    name: str
    cu_seqlens: np.ndarray      # int32 [nseq + 1]
    hq: int
    hkv: int
    head_dim: int
    block_size: int
    topk: int
    scale: float
    q: np.ndarray               # [T, hq, d]
    k: np.ndarray               # [T, hkv, d]
    v: np.ndarray               # [T, hkv, d]
    dout: np.ndarray | None     # [T, hq, d]
    block_idx: np.ndarray       # int32 [T, hkv, topk]
    seed: int

    @property
    def T(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def nseq(self) -> int:
        return len(self.cu_seqlens) - 1

    @property
    def max_seqlen(self) -> int:
        cu = self.cu_seqlens.astype(np.int64)
        return int((cu[1:] - cu[:-1]).max()) if self.nseq else 0


def make_problem(lengths, hq: int, hkv: int, head_dim: int = 128, block_size: int = 64,
                 topk: int = 16, seed: int = 0, with_dout: bool = True,
                 name: str = "custom", block_idx: np.ndarray | None = None) -> Problem:
    cu = cu_seqlens_from_lengths(lengths)
    T = int(cu[-1])
    rng = np.random.Generator(np.random.PCG64(seed))
    draw = lambda shape: bf16_round(rng.standard_normal(shape, dtype=np.float32), inplace=True)
    q = draw((T, hq, head_dim))
    k = draw((T, hkv, head_dim))
    v = draw((T, hkv, head_dim))
    dout = draw((T, hq, head_dim)) if with_dout else None
    if block_idx is None:
        block_idx = make_block_idx(cu, hkv, topk, block_size, seed)
    return Problem(name=name, cu_seqlens=cu, hq=hq, hkv=hkv, head_dim=head_dim,
                   block_size=block_size, topk=topk, scale=1.0 / math.sqrt(head_dim),
                   q=q, k=k, v=v, dout=dout, block_idx=block_idx, seed=seed)


# The workloads.  Seeds: workload n uses seed n; every sweep point uses seed 4.
WORKLOADS = {
    "tiny_t2k_g1_k8": dict(lengths=[2048], hq=4, hkv=4, block_size=64, topk=8, seed=1),
    "fwd_t32k_hq32_g4_k16": dict(lengths=[32768], hq=32, hkv=8, block_size=64, topk=16, seed=2),
    "varlen_64k_32k_g1_k16": dict(lengths=[65536, 32768], hq=4, hkv=4, block_size=64, topk=16, seed=3),
    "train_t32k_hq64_g8_k16": dict(lengths=[32768], hq=64, hkv=8, block_size=64, topk=16, seed=5),
    # half of the headline sequence, same heads: the profiling capture size
    "prof_t32k_hq16_g4_k16": dict(lengths=[32768], hq=16, hkv=4, block_size=64, topk=16, seed=4),
}


def sweep_workload(group: int, block_size: int, topk: int) -> dict:
    """One point of the T=65536, Hkv=4 sweep."""
    return dict(lengths=[65536], hq=4 * group, hkv=4, block_size=block_size, topk=topk, seed=4)


SWEEP_POINTS = [(g, bs, k) for g in (1, 2, 4, 8, 16) for bs in (64, 128) for k in (8, 16, 32)]
for _g, _bs, _k in SWEEP_POINTS:
    WORKLOADS[f"sweep_t64k_g{_g}_bs{_bs}_k{_k}"] = sweep_workload(_g, _bs, _k)

# The headline point: T=65536, group 4, block 64, topk 16.
HEADLINE = "sweep_t64k_g4_bs64_k16"


def workload(name: str, with_dout: bool = True) -> Problem:
    spec = dict(WORKLOADS[name])
    return make_problem(name=name, with_dout=with_dout, head_dim=128, **spec)

