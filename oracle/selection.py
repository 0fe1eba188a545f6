"""fp64 CPU oracle of the block-selection step -- TEST INFRASTRUCTURE.

The step that produces ``block_idx`` for the selected-block attention: compressed
keys and values, attention over them, per-block importance scores and the top-k
choice.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py`` may import this module; the product path never does.

What the pages fix: the quick start of the "Relaxed-System-Lab/Flash-Sparse-Attention"
project page builds the module with kernel_size 32, kernel_stride 16, block_size 64,
topk 16, init_blocks 1 and local_blocks 2.  They print no formula for any of the
steps below, so each step takes the plainest reading that those parameters support
(all of them listed with the other readings of the pages):

* compression: compressed block c of a sequence covers its tokens
  [c * stride, c * stride + kernel_size); there are floor((L - kernel_size) / stride)
  + 1 of them (none when L < kernel_size).  Its key and value are the means of the
  covered keys and values (a parameter-free stand-in for a learned pooling).
* compressed attention: the token at local position i sees compressed block c when
  the block ends at or before it, c * stride + kernel_size - 1 <= i; probabilities
  are the softmax of scale * q . k_c over the blocks it sees; a token that sees none
  gets probability 0 everywhere, output 0 and LSE -inf.
* block scores: the score of selection block b for (token, KV head g) is the sum,
  over the G query heads of g and over the compressed blocks whose span intersects
  [b * block_size, (b + 1) * block_size), of the compressed probabilities.
* top-k: blocks 0 .. init_blocks - 1 and the local blocks qb, qb - 1, ..,
  qb - local_blocks + 1 (those in [0, qb]) are always chosen, in that order; the
  remaining slots take the other blocks b <= qb by descending score, ties to the
  lower block; unused slots are -1.

Parity status (``tests/test_selection_oracle.py``): every function is pinned --
compression by closed forms and a cumulative-sum formulation, the compressed
attention against torch float64 SDPA under an explicit mask, the scores by closed
forms (a single visible compressed block, the mass conservation count) and a dense
overlap-matrix product, the top-k against a full sort and by the order invariants.
"""
from __future__ import annotations

import math

import numpy as np


def num_compressed(L: int, kernel_size: int, stride: int) -> int:
    """Compressed blocks of a sequence of L tokens."""
    return 0 if L < kernel_size else (L - kernel_size) // stride + 1


def compress_kv(k, v, cu_seqlens, kernel_size: int = 32, stride: int = 16):
    """Mean-pooled compressed keys and values.

    Returns (k_cmp [C, hkv, d], v_cmp [C, hkv, d], cu_cmp int64 [nseq + 1]) with the
    compressed blocks of sequence s at rows cu_cmp[s] .. cu_cmp[s + 1] - 1."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    nseq = len(cu) - 1
    counts = [num_compressed(int(cu[s + 1] - cu[s]), kernel_size, stride) for s in range(nseq)]
    cu_cmp = np.zeros(nseq + 1, dtype=np.int64)
    cu_cmp[1:] = np.cumsum(counts)
    hkv, d = k.shape[1], k.shape[2]
    k_cmp = np.zeros((int(cu_cmp[-1]), hkv, d))
    v_cmp = np.zeros((int(cu_cmp[-1]), hkv, d))
    for s in range(nseq):
        a = int(cu[s])
        for c in range(counts[s]):
            lo = a + c * stride
            k_cmp[cu_cmp[s] + c] = k[lo:lo + kernel_size].astype(np.float64).mean(axis=0)
            v_cmp[cu_cmp[s] + c] = v[lo:lo + kernel_size].astype(np.float64).mean(axis=0)
    return k_cmp, v_cmp, cu_cmp


def compressed_attention(q, k_cmp, v_cmp, cu_seqlens, cu_cmp, scale: float,
                         kernel_size: int = 32, stride: int = 16):
    """Attention of every query over the compressed blocks it sees.

    Returns (out [T, hq, d], lse [T, hq], probs): probs[s] is the [L_s, hq, C_s]
    probability array of sequence s (rows of tokens that see no block are 0)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T, hq, d = q.shape
    hkv = k_cmp.shape[1]
    G = hq // hkv
    out = np.zeros((T, hq, d))
    lse = np.full((T, hq), -np.inf)
    probs = []
    for s in range(len(cu) - 1):
        a, L = int(cu[s]), int(cu[s + 1] - cu[s])
        c0, C = int(cu_cmp[s]), int(cu_cmp[s + 1] - cu_cmp[s])
        ps = np.zeros((L, hq, C))
        for i in range(L):
            nvis = 0 if i < kernel_size - 1 else min(C, (i - kernel_size + 1) // stride + 1)
            if nvis == 0:
                continue
            for h in range(hq):
                g = h // G
                sc = scale * (k_cmp[c0:c0 + nvis, g] @ q[a + i, h].astype(np.float64))
                m = sc.max()
                w = np.exp(sc - m)
                tot = w.sum()
                lse[a + i, h] = m + math.log(tot)
                ps[i, h, :nvis] = w / tot
                out[a + i, h] = ps[i, h, :nvis] @ v_cmp[c0:c0 + nvis, g]
        probs.append(ps)
    return out, lse, probs


def block_scores(probs, cu_seqlens, hkv: int, block_size: int = 64, kernel_size: int = 32,
                 stride: int = 16):
    """Importance of each selection block: a list over sequences of [L_s, hkv, NB_s]
    arrays, summing the compressed probabilities of the group's heads over the
    compressed blocks whose span meets the selection block."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    out = []
    for s, ps in enumerate(probs):
        L = int(cu[s + 1] - cu[s])
        hq, C = ps.shape[1], ps.shape[2]
        G = hq // hkv
        nb = (L + block_size - 1) // block_size
        sc = np.zeros((L, hkv, nb))
        for c in range(C):
            first, last = c * stride, c * stride + kernel_size - 1
            for b in range(first // block_size, min(last // block_size, nb - 1) + 1):
                for g in range(hkv):
                    sc[:, g, b] += ps[:, g * G:(g + 1) * G, c].sum(axis=1)
        out.append(sc)
    return out


def select_topk(scores, cu_seqlens, topk: int = 16, block_size: int = 64, init_blocks: int = 1,
                local_blocks: int = 2):
    """block_idx int32 [T, hkv, topk]: forced initial and local blocks, then the best
    scored of the other causal blocks (ties to the lower block), -1 padded."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T = int(cu[-1])
    hkv = scores[0].shape[1] if scores else 1
    out = np.full((T, hkv, topk), -1, dtype=np.int32)
    for s, sc in enumerate(scores):
        a, L = int(cu[s]), int(cu[s + 1] - cu[s])
        for i in range(L):
            qb = i // block_size
            forced = [b for b in range(init_blocks) if b <= qb]
            forced += [b for b in range(qb, qb - local_blocks, -1) if b >= 0 and b not in forced]
            forced = forced[:topk]
            rest = [b for b in range(qb + 1) if b not in forced]
            for g in range(hkv):
                # descending score, ascending block on ties
                order = sorted(rest, key=lambda b: (-sc[i, g, b], b))
                row = forced + order[:topk - len(forced)]
                out[a + i, g, :len(row)] = row
    return out


def select(q, k, v, cu_seqlens, scale: float, topk: int = 16, block_size: int = 64,
           kernel_size: int = 32, stride: int = 16, init_blocks: int = 1, local_blocks: int = 2):
    """The whole selection step: (block_idx [T, hkv, topk], compressed output [T, hq, d],
    compressed LSE [T, hq])."""
    k_cmp, v_cmp, cu_cmp = compress_kv(k, v, cu_seqlens, kernel_size, stride)
    o_cmp, lse_cmp, probs = compressed_attention(q, k_cmp, v_cmp, cu_seqlens, cu_cmp, scale,
                                                 kernel_size, stride)
    sc = block_scores(probs, cu_seqlens, k.shape[1], block_size, kernel_size, stride)
    bidx = select_topk(sc, cu_seqlens, topk, block_size, init_blocks, local_blocks)
    return bidx, o_cmp, lse_cmp
