"""Pins for the fp64 oracle of threshold-pruned block attention (CPU only)."""
import numpy as np
import torch

import nsa_inputs as ni
import oracle
from oracle import bsfa

BS = 16


def _problem(lengths, hq, hkv, seed):
    return ni.make_problem(lengths, hq=hq, hkv=hkv, head_dim=16, block_size=BS, topk=4, seed=seed)


def test_no_threshold_is_dense_causal_attention():
    p = _problem([70, 33], hq=4, hkv=2, seed=1)
    o, l, kept = bsfa.bsfa_fwd(p.q, p.k, p.v, p.cu_seqlens, BS, p.scale, -np.inf)
    for s in range(2):
        a, b = int(p.cu_seqlens[s]), int(p.cu_seqlens[s + 1])
        L = b - a
        assert np.all(kept[s] == (np.arange((L + BS - 1) // BS)[None, None, :] <=
                                  (np.arange(L) // BS)[:, None, None]))
        qs = torch.from_numpy(p.q[a:b].astype(np.float64)).permute(1, 0, 2)
        ks = torch.from_numpy(p.k[a:b].astype(np.float64)).repeat_interleave(2, 1).permute(1, 0, 2)
        vs = torch.from_numpy(p.v[a:b].astype(np.float64)).repeat_interleave(2, 1).permute(1, 0, 2)
        ro = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, is_causal=True, scale=p.scale)
        np.testing.assert_allclose(o[a:b], ro.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
        sc = (qs @ ks.transpose(1, 2)) * p.scale
        sc = sc.masked_fill(~torch.ones(L, L, dtype=torch.bool).tril(), float("-inf"))
        np.testing.assert_allclose(l[a:b], torch.logsumexp(sc, -1).permute(1, 0).numpy(), rtol=0,
                                   atol=1e-12)


def test_equals_selected_attention_on_the_kept_blocks():
    # one query head per KV head: the kept blocks of a row are a selected-block index
    p = _problem([150, 61], hq=3, hkv=3, seed=2)
    tau = np.array([0.2, 0.5, 0.9])
    o, l, kept = bsfa.bsfa_fwd(p.q, p.k, p.v, p.cu_seqlens, BS, p.scale, tau)
    nbmax = max(kk.shape[2] for kk in kept)
    bi = np.full((p.q.shape[0], 3, nbmax), -1, dtype=np.int32)
    frac = []
    for s in range(2):
        a = int(p.cu_seqlens[s])
        for i in range(kept[s].shape[0]):
            for h in range(3):
                blocks = np.nonzero(kept[s][i, h])[0]
                bi[a + i, h, :len(blocks)] = blocks
                frac.append(len(blocks) / (i // BS + 1))
    assert 0.2 < np.mean(frac) < 0.95          # the thresholds prune a real share of blocks
    ro, rl = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, bi, BS, p.scale)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, rl, rtol=0, atol=1e-12)


def test_kept_blocks_brute_force_and_extremes():
    p = _problem([90], hq=4, hkv=1, seed=3)
    tau = np.array([-0.1, 0.0, 0.3, 0.6])
    _, _, kept = bsfa.bsfa_fwd(p.q, p.k, p.v, p.cu_seqlens, BS, p.scale, tau)
    S = p.scale * np.einsum("thd,jd->thj", p.q.astype(np.float64), p.k[:, 0].astype(np.float64))
    for t in range(90):
        for h in range(4):
            for b in range(6):
                keys = [j for j in range(b * BS, min(b * BS + BS, 90)) if j <= t]
                want = bool(keys) and max(S[t, h, j] for j in keys) >= tau[h]
                assert kept[0][t, h, b] == want
    # a threshold above every score keeps nothing: O = 0, LSE = -inf
    o, l, kept = bsfa.bsfa_fwd(p.q, p.k, p.v, p.cu_seqlens, BS, p.scale, 1e9)
    assert not kept[0].any() and np.all(o == 0) and np.all(np.isneginf(l))
