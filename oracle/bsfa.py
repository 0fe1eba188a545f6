"""fp64 CPU oracle of threshold-pruned block attention -- TEST INFRASTRUCTURE.

Block Sparse Flash Attention as the "Block Sparse Flash Attention" news pages (the
aiqbench analysis and the marsel.app article, "How it works") describe it: every
query-key score is computed exactly; for each query and each key block the block's
largest score is compared with a calibrated threshold, and blocks below it are
skipped (their values are neither loaded nor multiplied).  Only ``tests/`` may import
this module; the product path never does.

The pages print no formula, so the plainest reading is taken (and listed with the
other readings of the pages):

* key blocks are the block_size-aligned blocks of each sequence (as in the selected
  attention), causal: key j <= query i;
* for query row (token i, query head h), block b is kept iff
  max_{j in b, j <= i} scale * q_i . k_j >= tau[h] (one threshold per query head; the
  calibration that sets it is not reproduced: thresholds are inputs);
* the output is softmax attention over the keys of the kept blocks only (a skipped
  block contributes to neither the numerator nor the normaliser); a row that keeps no
  block gets O = 0 and LSE = -inf.

Parity status (``tests/test_bsfa_oracle.py``): pinned -- tau = -inf against torch
float64 SDPA with a causal mask; equal, for one query head per KV head, to the
selected-attention oracle given the kept blocks as its index; the kept set against
a brute-force loop; thresholds above every score keep nothing.
"""
from __future__ import annotations

import math

import numpy as np


def bsfa_fwd(q, k, v, cu_seqlens, block_size: int, scale: float, tau):
    """Returns (out [T, hq, d], lse [T, hq], kept): kept[s] is the boolean [L_s, hq, NB_s]
    array of kept blocks of sequence s."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    tau = np.broadcast_to(np.asarray(tau, dtype=np.float64), (hq,))
    out = np.zeros((T, hq, d))
    lse = np.full((T, hq), -np.inf)
    kept_all = []
    for s in range(len(cu) - 1):
        a, L = int(cu[s]), int(cu[s + 1] - cu[s])
        nb = (L + block_size - 1) // block_size
        kept = np.zeros((L, hq, nb), dtype=bool)
        for i in range(L):
            qb = i // block_size
            for h in range(hq):
                g = h // G
                # exact scores of every causal key of the row
                sc = scale * (k[a:a + i + 1, g].astype(np.float64) @ q[a + i, h].astype(np.float64))
                keys = []
                for b in range(qb + 1):
                    lo, hi = b * block_size, min((b + 1) * block_size, i + 1)
                    if sc[lo:hi].max() >= tau[h]:
                        kept[i, h, b] = True
                        keys.extend(range(lo, hi))
                if not keys:
                    continue
                ks = np.asarray(keys)
                m = sc[ks].max()
                w = np.exp(sc[ks] - m)
                lse[a + i, h] = m + math.log(w.sum())
                out[a + i, h] = (w / w.sum()) @ v[a + ks, g].astype(np.float64)
        kept_all.append(kept)
    return out, lse, kept_all
