"""Pins for the fp64 oracle of the block-selection step (CPU only).

Each check ties a step to something other than its own code: closed forms, a
cumulative-sum or overlap-matrix formulation, torch float64 SDPA under an explicit
mask, a full sort by numpy, and the order invariants of the top-k rule.
"""
import numpy as np
import pytest
import torch

import nsa_inputs as ni
import oracle
from oracle import selection as sel

KS, STRIDE, BS = 32, 16, 64


def _problem(lengths, hq=4, hkv=2, d=16, seed=0):
    return ni.make_problem(lengths, hq=hq, hkv=hkv, head_dim=d, block_size=BS, topk=4, seed=seed)


def test_num_compressed_closed_forms():
    assert [sel.num_compressed(L, KS, STRIDE) for L in (0, 31, 32, 47, 48, 64, 1000)] == \
        [0, 0, 1, 1, 2, 3, 61]


def test_compress_closed_forms_and_prefix_sums():
    cu = ni.cu_seqlens_from_lengths([100, 31, 64])
    T = int(cu[-1])
    # constant keys pool to themselves; a ramp k[t] = local t pools to 16 c + 15.5
    k = np.full((T, 2, 8), 3.25)
    v = np.zeros((T, 2, 8))
    for s in range(3):
        v[cu[s]:cu[s + 1]] = np.arange(cu[s + 1] - cu[s])[:, None, None]
    kc, vc, cuc = sel.compress_kv(k, v, cu, KS, STRIDE)
    assert list(cuc) == [0, 5, 5, 8]
    assert np.all(kc == 3.25)
    np.testing.assert_allclose(vc[0:5, 0, 0], 16 * np.arange(5) + 15.5, rtol=0, atol=1e-12)
    np.testing.assert_allclose(vc[5:8, 1, 3], 16 * np.arange(3) + 15.5, rtol=0, atol=1e-12)
    # random values against window sums taken from prefix sums
    p = _problem([200, 50], seed=1)
    kc, vc, cuc = sel.compress_kv(p.k, p.v, p.cu_seqlens, KS, STRIDE)
    for s in range(2):
        a, L = int(p.cu_seqlens[s]), int(p.cu_seqlens[s + 1] - p.cu_seqlens[s])
        ps = np.concatenate([np.zeros((1, 2, 16)), np.cumsum(p.k[a:a + L].astype(np.float64), 0)])
        for c in range(sel.num_compressed(L, KS, STRIDE)):
            want = (ps[c * STRIDE + KS] - ps[c * STRIDE]) / KS
            np.testing.assert_allclose(kc[cuc[s] + c], want, rtol=0, atol=1e-12)


def test_compressed_attention_matches_masked_sdpa():
    p = _problem([300, 20, 90], hq=8, hkv=2, seed=2)
    kc, vc, cuc = sel.compress_kv(p.k, p.v, p.cu_seqlens, KS, STRIDE)
    out, lse, probs = sel.compressed_attention(p.q, kc, vc, p.cu_seqlens, cuc, p.scale, KS, STRIDE)
    G = 4
    for s in range(3):
        a, L = int(p.cu_seqlens[s]), int(p.cu_seqlens[s + 1] - p.cu_seqlens[s])
        c0, C = int(cuc[s]), int(cuc[s + 1] - cuc[s])
        i = np.arange(L)[:, None]
        c = np.arange(C)[None, :]
        vis = c * STRIDE + KS - 1 <= i                       # [L, C]
        rows = vis.any(axis=1)
        # tokens that see no compressed block: zero output, -inf LSE, zero probabilities
        assert np.all(out[a:a + L][~rows] == 0) and np.all(np.isneginf(lse[a:a + L][~rows]))
        assert np.all(probs[s][~rows] == 0)
        if C == 0 or not rows.any():
            continue
        qs = torch.from_numpy(p.q[a:a + L][rows].astype(np.float64)).permute(1, 0, 2)
        ks = torch.from_numpy(kc[c0:c0 + C]).repeat_interleave(G, 1).permute(1, 0, 2)
        vs = torch.from_numpy(vc[c0:c0 + C]).repeat_interleave(G, 1).permute(1, 0, 2)
        mask = torch.from_numpy(vis[rows])
        ro = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, attn_mask=mask,
                                                              scale=p.scale)
        np.testing.assert_allclose(out[a:a + L][rows], ro.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
        sc = (qs @ ks.transpose(1, 2)) * p.scale
        rl = torch.logsumexp(sc.masked_fill(~mask, float("-inf")), dim=-1).permute(1, 0).numpy()
        np.testing.assert_allclose(lse[a:a + L][rows], rl, rtol=0, atol=1e-12)
        np.testing.assert_allclose(probs[s][rows].sum(axis=2), 1.0, rtol=0, atol=1e-12)


def test_single_visible_block_closed_form():
    # tokens 31 .. 46 see exactly compressed block 0: p = 1, O = v_cmp[0],
    # LSE = scale q . k_cmp[0], and the score of selection block 0 is G
    p = _problem([64], hq=4, hkv=1, seed=3)
    kc, vc, cuc = sel.compress_kv(p.k, p.v, p.cu_seqlens, KS, STRIDE)
    out, lse, probs = sel.compressed_attention(p.q, kc, vc, p.cu_seqlens, cuc, p.scale, KS, STRIDE)
    sc = sel.block_scores(probs, p.cu_seqlens, 1, BS, KS, STRIDE)[0]
    for t in range(31, 47):
        for h in range(4):
            np.testing.assert_allclose(out[t, h], vc[0, 0], rtol=0, atol=1e-12)
            assert abs(lse[t, h] - p.scale * float(kc[0, 0] @ p.q[t, h].astype(np.float64))) < 1e-12
        assert sc[t, 0, 0] == pytest.approx(4.0, abs=1e-12)
    assert np.all(sc[:31] == 0)


def test_block_scores_overlap_matrix_and_mass():
    p = _problem([400, 130], hq=6, hkv=2, seed=4)
    kc, vc, cuc = sel.compress_kv(p.k, p.v, p.cu_seqlens, KS, STRIDE)
    _, _, probs = sel.compressed_attention(p.q, kc, vc, p.cu_seqlens, cuc, p.scale, KS, STRIDE)
    scores = sel.block_scores(probs, p.cu_seqlens, 2, BS, KS, STRIDE)
    for s, (ps, sc) in enumerate(zip(probs, scores)):
        L, _, C = ps.shape
        nb = sc.shape[2]
        # overlap matrix by interval intersection: [16c, 16c + 31] meets [64b, 64b + 63]
        c = np.arange(C)[:, None]
        b = np.arange(nb)[None, :]
        A = (np.maximum(c * STRIDE, b * BS) <= np.minimum(c * STRIDE + KS - 1, b * BS + BS - 1))
        grp = ps.reshape(L, 2, 3, C).sum(axis=2)                       # [L, hkv, C]
        np.testing.assert_allclose(sc, grp @ A.astype(np.float64), rtol=0, atol=1e-12)
        # mass: every probability is counted once per selection block its span meets
        nmeet = A.sum(axis=1)                                          # 1 or 2
        vis = ps.sum(axis=2)[:, 0] > 0
        want = (ps[:, :3, :] * nmeet).sum(axis=(1, 2))
        np.testing.assert_allclose(sc[:, 0, :].sum(axis=1), want, rtol=0, atol=1e-11)
        assert np.all(sc[vis].sum(axis=2) >= 3 - 1e-12)                # >= G where anything is seen


@pytest.mark.parametrize("topk,init,local", [(16, 1, 2), (5, 1, 2), (3, 1, 2), (6, 2, 3), (1, 1, 2)])
def test_topk_against_full_sort_and_invariants(topk, init, local):
    rng = np.random.default_rng(5)
    cu = ni.cu_seqlens_from_lengths([700, 65, 0, 130])
    scores = []
    for s in range(len(cu) - 1):
        L = int(cu[s + 1] - cu[s])
        nb = (L + BS - 1) // BS
        x = rng.random((L, 2, nb))
        x[:, :, ::3] = np.round(x[:, :, ::3], 1)                      # plant ties
        scores.append(x)
    bi = sel.select_topk(scores, cu, topk, BS, init, local)
    for s in range(len(cu) - 1):
        a, L = int(cu[s]), int(cu[s + 1] - cu[s])
        for i in range(L):
            qb = i // BS
            forced = []
            for bb in list(range(init)) + list(range(qb, qb - local, -1)):
                if 0 <= bb <= qb and bb not in forced:
                    forced.append(bb)
            forced = forced[:topk]
            for g in range(2):
                row = [int(x) for x in bi[a + i, g] if x >= 0]
                assert row[:len(forced)] == forced
                assert len(row) == len(set(row)) == min(topk, qb + 1)
                assert all(0 <= bb <= qb for bb in row)
                assert np.all(bi[a + i, g, len(row):] == -1)
                # the rest: numpy's full sort by (-score, block) over the free blocks
                free = np.array([bb for bb in range(qb + 1) if bb not in forced], dtype=np.int64)
                if len(free):
                    order = free[np.lexsort((free, -scores[s][i, g, free]))]
                    assert row[len(forced):] == [int(x) for x in order[:topk - len(forced)]]


def test_selection_feeds_the_attention_oracle():
    # enough slots for every causal block: the chosen index makes the selected attention
    # dense causal attention, whatever the scores
    p = _problem([260, 70], hq=4, hkv=2, d=16, seed=6)
    bi, _, _ = sel.select(p.q, p.k, p.v, p.cu_seqlens, p.scale, topk=5, block_size=BS)
    for s in range(2):
        a, L = int(p.cu_seqlens[s]), int(p.cu_seqlens[s + 1] - p.cu_seqlens[s])
        for i in range(L):
            assert sorted(int(x) for x in bi[a + i, 0] if x >= 0) == list(range(i // BS + 1))
    o, l = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, bi, BS, p.scale)
    o2, l2 = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens,
                        np.tile(np.arange(5, dtype=np.int32), (p.q.shape[0], 2, 1)), BS, p.scale)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, l2, rtol=0, atol=1e-12)


def test_forced_slots_agree_with_the_index_generator():
    # the synthetic index rule starts every row with 0, qb, qb - 1 (deduplicated): the
    # forced part of the top-k with init_blocks 1 and local_blocks 2
    cu = ni.cu_seqlens_from_lengths([500])
    gen = ni.make_block_idx(cu, 2, 16, BS, seed=7)
    scores = [np.zeros((500, 2, 8))]
    bi = sel.select_topk(scores, cu, 16, BS, 1, 2)
    for t in range(500):
        qb = t // BS
        nforced = min(3, qb + 1)
        assert np.array_equal(bi[t, :, :nforced], gen[t, :, :nforced])
