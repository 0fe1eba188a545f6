"""Pins for the fp64 oracle (CPU only).

Each check ties the oracle to something other than itself: a library routine
(torch float64 SDPA / autograd), a differently formulated brute force, finite
differences, hand-derived closed forms, or an invariant of the definition.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import nsa_inputs as ni
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _all_blocks_idx(cu, hkv, block_size, topk, rng=None):
    """block_idx that selects every block of the token's sequence (any order)."""
    cu = np.asarray(cu, dtype=np.int64)
    T = int(cu[-1])
    out = np.full((T, hkv, topk), -1, dtype=np.int32)
    for s in range(len(cu) - 1):
        L = int(cu[s + 1] - cu[s])
        nb = (L + block_size - 1) // block_size
        assert nb <= topk
        for t in range(int(cu[s]), int(cu[s + 1])):
            for g in range(hkv):
                row = np.full(topk, -1, dtype=np.int32)
                row[:nb] = np.arange(nb)
                if rng is not None:
                    rng.shuffle(row)
                out[t, g] = row
    return out


def _sdpa_causal_f64(q, k, v, cu, scale):
    """Dense causal attention per sequence with torch float64 SDPA (GQA expanded)."""
    T, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    out = np.zeros((T, hq, d))
    lse = np.zeros((T, hq))
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        qs = torch.from_numpy(q[a:b].astype(np.float64)).permute(1, 0, 2)          # [hq, L, d]
        ks = torch.from_numpy(k[a:b].astype(np.float64)).repeat_interleave(G, 1).permute(1, 0, 2)
        vs = torch.from_numpy(v[a:b].astype(np.float64)).repeat_interleave(G, 1).permute(1, 0, 2)
        o = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, is_causal=True, scale=scale)
        out[a:b] = o.permute(1, 0, 2).numpy()
        sc = (qs @ ks.transpose(1, 2)) * scale
        L = b - a
        mask = torch.ones(L, L, dtype=torch.bool).tril()
        sc = sc.masked_fill(~mask, float("-inf"))
        lse[a:b] = torch.logsumexp(sc, dim=-1).permute(1, 0).numpy()
    return out, lse


def _brute_mask(cu, block_idx, block_size):
    """Explicit [T, hkv, T] boolean mask built from block_idx (a second formulation)."""
    cu = np.asarray(cu, dtype=np.int64)
    T, hkv, topk = block_idx.shape
    M = np.zeros((T, hkv, T), dtype=bool)
    seq = np.searchsorted(cu, np.arange(T), side="right") - 1
    for t in range(T):
        for g in range(hkv):
            for j in range(T):
                if seq[j] != seq[t] or j > t:
                    continue
                blk = (j - cu[seq[j]]) // block_size
                if blk in set(int(x) for x in block_idx[t, g]):
                    M[t, g, j] = True
    return M


def _brute_fwd(q, k, v, M, scale):
    T, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    out = np.zeros((T, hq, d))
    lse = np.full((T, hq), -np.inf)
    for t in range(T):
        for h in range(hq):
            g = h // G
            keys = np.nonzero(M[t, g])[0]
            if len(keys) == 0:
                continue
            s = scale * (k[keys, g].astype(np.float64) @ q[t, h].astype(np.float64))
            mx = s.max()
            w = np.exp(s - mx)
            lse[t, h] = mx + math.log(w.sum())
            out[t, h] = (w / w.sum()) @ v[keys, g].astype(np.float64)
    return out, lse


# --------------------------------------------------------------------------- forward pins

@pytest.mark.parametrize("lengths,hq,hkv,bs,d", [([96], 4, 2, 16, 32), ([40, 70, 1, 17], 2, 1, 16, 32),
                                                ([130], 8, 2, 32, 32), ([70], 2, 1, 32, 64),
                                                ([70], 2, 2, 32, 128), ([45], 4, 1, 16, 256)])
def test_fwd_dense_causal_equals_sdpa(lengths, hq, hkv, bs, d):
    """topk covering every causal block reduces to dense causal attention (any head dim)."""
    cu = ni.cu_seqlens_from_lengths(lengths)
    nb = max((L + bs - 1) // bs for L in lengths)
    p = ni.make_problem(lengths, hq=hq, hkv=hkv, head_dim=d, block_size=bs, topk=nb + 1, seed=11,
                        block_idx=_all_blocks_idx(cu, hkv, bs, nb + 1, np.random.default_rng(3)))
    o, l = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, bs, p.scale)
    ro, rl = _sdpa_causal_f64(p.q, p.k, p.v, p.cu_seqlens, p.scale)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, rl, rtol=0, atol=1e-12)


def test_fwd_brute_force_mask():
    """Random selections vs an explicit T x T mask and dense masked softmax."""
    p = ni.make_problem([70, 58], hq=4, hkv=2, head_dim=16, block_size=8, topk=4, seed=5)
    # add out-of-range, future and -1 entries in random places
    bi = p.block_idx.copy()
    rng = np.random.default_rng(0)
    for _ in range(60):
        t, g, j = rng.integers(0, p.T), rng.integers(0, 2), rng.integers(0, 4)
        bi[t, g, j] = rng.choice([-1, 50, 3, 9])
    o, l = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, bi, 8, p.scale)
    M = _brute_mask(p.cu_seqlens, bi, 8)
    ro, rl = _brute_fwd(p.q, p.k, p.v, M, p.scale)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, rl, rtol=0, atol=1e-12)


def test_fwd_index_order_invariance():
    p = ni.make_problem([300], hq=4, hkv=2, head_dim=32, block_size=16, topk=6, seed=2)
    rng = np.random.default_rng(9)
    bi2 = p.block_idx.copy()
    for t in range(p.T):
        for g in range(2):
            rng.shuffle(bi2[t, g])
    o1, l1 = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, 16, p.scale)
    o2, l2 = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, bi2, 16, p.scale)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_fwd_weights_sum_to_one():
    """V = one-hot per key makes O the weight vector: it sums to 1, is >= 0 and is
    zero off the selected causal keys; constant V gives O = V."""
    T, d = 100, 128
    p = ni.make_problem([T], hq=2, hkv=1, head_dim=d, block_size=8, topk=5, seed=4)
    v = np.zeros((T, 1, d), dtype=np.float32)
    v[np.arange(T), 0, np.arange(T)] = 1.0
    o, _ = oracle.fwd(p.q, p.k, v, p.cu_seqlens, p.block_idx, 8, p.scale)
    np.testing.assert_allclose(o.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (o >= 0).all()
    M = _brute_mask(p.cu_seqlens, p.block_idx, 8)
    for h in range(2):
        assert (o[:, h, :T][~M[:, 0, :]] == 0).all()
    vc = np.full((T, 1, d), 0.75, dtype=np.float32)
    o2, _ = oracle.fwd(p.q, p.k, vc, p.cu_seqlens, p.block_idx, 8, p.scale)
    np.testing.assert_allclose(o2, 0.75, rtol=0, atol=1e-13)


def test_fwd_closed_forms():
    p = ni.make_problem([200], hq=4, hkv=2, head_dim=32, block_size=16, topk=5, seed=8)
    o, l = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, 16, p.scale)
    # token 0 attends only key 0
    for h in range(4):
        g = h // 2
        np.testing.assert_allclose(o[0, h], p.v[0, g], rtol=0, atol=1e-15)
        assert abs(l[0, h] - p.scale * float(np.dot(p.q[0, h].astype(np.float64),
                                                     p.k[0, g].astype(np.float64)))) < 1e-13
    # K = 0: O is the mean of the attended V and LSE = ln |J|
    k0 = np.zeros_like(p.k)
    o, l = oracle.fwd(p.q, k0, p.v, p.cu_seqlens, p.block_idx, 16, p.scale)
    M = _brute_mask(p.cu_seqlens, p.block_idx, 16)
    for t in (5, 17, 63, 199):
        for h in range(4):
            g = h // 2
            keys = np.nonzero(M[t, g])[0]
            np.testing.assert_allclose(o[t, h], p.v[keys, g].astype(np.float64).mean(0), atol=1e-13)
            assert abs(l[t, h] - math.log(len(keys))) < 1e-13


def test_fwd_hand_worked_example():
    ex = json.load(open(os.path.join(GOLDEN, "hand_worked_example.json")))
    env = {"e": math.e, "ln": math.log}
    q = np.array(ex["q"], dtype=np.float32)
    k = np.array(ex["k"], dtype=np.float32)
    v = np.array(ex["v"], dtype=np.float32)
    bi = np.array(ex["block_idx"], dtype=np.int32)
    o, l = oracle.fwd(q, k, v, np.array(ex["cu_seqlens"], np.int32), bi, ex["block_size"], ex["scale"])
    for c in ex["expected"]:
        t, h = c["token"], c["head"]
        want_o = [eval(s, {"__builtins__": {}}, env) for s in c["O"]]
        want_l = eval(c["LSE"], {"__builtins__": {}}, env)
        np.testing.assert_allclose(o[t, h], want_o, rtol=0, atol=1e-14)
        assert abs(l[t, h] - want_l) < 1e-14


def test_fwd_empty_selection():
    """A row with no valid block (all -1, or only out-of-range) gives O = 0, LSE = -inf."""
    p = ni.make_problem([64], hq=2, hkv=1, head_dim=16, block_size=16, topk=3, seed=1)
    bi = p.block_idx.copy()
    bi[10, 0] = [-1, -1, -1]
    bi[20, 0] = [-1, 7, -5]
    o, l = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, bi, 16, p.scale)
    for t in (10, 20):
        assert (o[t] == 0).all() and np.isneginf(l[t]).all()


def test_fwd_token_subset_matches_full():
    p = ni.make_problem([120, 77], hq=4, hkv=2, head_dim=32, block_size=16, topk=4, seed=6)
    o, l = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, 16, p.scale)
    toks = np.array([0, 5, 119, 120, 150, 196])
    o2, l2 = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, 16, p.scale, tokens=toks)
    assert np.array_equal(o[toks], o2) and np.array_equal(l[toks], l2)


# -------------------------------------------------------------------------- backward pins

def _loss(p, q, k, v, bi, bs):
    o, _ = oracle.fwd(q, k, v, p.cu_seqlens, bi, bs, p.scale)
    return float((o * p.dout.astype(np.float64)).sum())


def test_bwd_finite_differences():
    """Central differences of L = sum(dO * O) along exactly representable directions."""
    p = ni.make_problem([48, 21], hq=4, hkv=2, head_dim=16, block_size=8, topk=3, seed=3)
    bs = 8
    dq, dk, dv = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, bs, p.scale)
    rng = np.random.default_rng(1)
    h = 2.0 ** -12
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        base = getattr(p, name)
        for _ in range(3):
            u = rng.choice([-1.0, 1.0], size=base.shape).astype(np.float32)
            plus, minus = base + np.float32(h) * u, base - np.float32(h) * u
            # the perturbation is exact in float32 for these bf16-valued inputs
            assert np.array_equal((plus - base).astype(np.float64), h * u.astype(np.float64))
            args = {"q": p.q, "k": p.k, "v": p.v}
            args[name] = plus
            lp = _loss(p, args["q"], args["k"], args["v"], p.block_idx, bs)
            args[name] = minus
            lm = _loss(p, args["q"], args["k"], args["v"], p.block_idx, bs)
            fd = (lp - lm) / (2 * h)
            an = float((grad * u.astype(np.float64)).sum())
            assert abs(fd - an) <= 2e-6 * max(1.0, abs(an)), (name, fd, an)


@pytest.mark.parametrize("d", [32, 64, 256])
def test_bwd_dense_causal_matches_autograd(d):
    lengths, hq, hkv, bs = [64, 37], 4, 2, 16
    cu = ni.cu_seqlens_from_lengths(lengths)
    nb = 4
    p = ni.make_problem(lengths, hq=hq, hkv=hkv, head_dim=d, block_size=bs, topk=nb + 2, seed=12,
                        block_idx=_all_blocks_idx(cu, hkv, bs, nb + 2, np.random.default_rng(5)))
    dq, dk, dv = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, bs, p.scale)
    G = hq // hkv
    q = torch.from_numpy(p.q.astype(np.float64)).requires_grad_()
    k = torch.from_numpy(p.k.astype(np.float64)).requires_grad_()
    v = torch.from_numpy(p.v.astype(np.float64)).requires_grad_()
    loss = 0
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        o = torch.nn.functional.scaled_dot_product_attention(
            q[a:b].permute(1, 0, 2), k[a:b].repeat_interleave(G, 1).permute(1, 0, 2),
            v[a:b].repeat_interleave(G, 1).permute(1, 0, 2), is_causal=True, scale=p.scale)
        loss = loss + (o.permute(1, 0, 2) * torch.from_numpy(p.dout[a:b].astype(np.float64))).sum()
    loss.backward()
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=0, atol=1e-11)


def test_bwd_sum_identities():
    """Rows of dS sum to zero (so dK summed over a head's keys is 0), and the weights
    of each row sum to one (so dV summed over keys equals dO summed over rows)."""
    p = ni.make_problem([150], hq=4, hkv=2, head_dim=32, block_size=16, topk=5, seed=13)
    dq, dk, dv = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, 16, p.scale)
    for g in range(2):
        assert np.abs(dk[:, g].sum(0)).max() < 1e-11
        want = p.dout[:, 2 * g:2 * g + 2].astype(np.float64).sum((0, 1))
        np.testing.assert_allclose(dv[:, g].sum(0), want, rtol=0, atol=1e-10)


def test_bwd_partial_entry_points_match_full():
    p = ni.make_problem([100, 60], hq=4, hkv=2, head_dim=32, block_size=16, topk=4, seed=14)
    dq, dk, dv = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, 16, p.scale)
    toks = np.array([0, 33, 99, 100, 159])
    dq2 = oracle.bwd_dq(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, 16, p.scale, toks)
    np.testing.assert_allclose(dq2, dq[toks], rtol=0, atol=1e-12)
    for g, key0, n in ((0, 0, 16), (1, 32, 16), (1, 96, 4), (0, 148, 12), (1, 100, 16)):
        dk2, dv2 = oracle.bwd_dkdv_keys(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, 16,
                                        p.scale, g, key0, n)
        np.testing.assert_allclose(dk2, dk[key0:key0 + n, g], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv2, dv[key0:key0 + n, g], rtol=0, atol=1e-12)


# ------------------------------------------------------------------------- inversion pins

def _brute_invert(cu, bi, bs):
    cu = np.asarray(cu, dtype=np.int64)
    T, hkv, topk = bi.shape
    nbs = [(int(cu[s + 1] - cu[s]) + bs - 1) // bs for s in range(len(cu) - 1)]
    offs, ents = [0], []
    for g in range(hkv):
        for s in range(len(cu) - 1):
            for b in range(nbs[s]):
                for t in range(int(cu[s]), int(cu[s + 1])):
                    qb = (t - int(cu[s])) // bs
                    for j in range(topk):
                        if bi[t, g, j] == b and b <= qb:
                            ents.append(t * 64 + j)
                offs.append(len(ents))
    return np.array(offs, dtype=np.int32), np.array(ents, dtype=np.int32)


def test_invert_brute_force():
    p = ni.make_problem([90, 33, 1, 64], hq=2, hkv=2, head_dim=8, block_size=16, topk=5, seed=21)
    bi = p.block_idx.copy()
    rng = np.random.default_rng(2)
    for _ in range(40):   # out-of-range / future / padding in random slots
        bi[rng.integers(0, p.T), rng.integers(0, 2), rng.integers(0, 5)] = rng.choice([-1, -3, 4, 99])
    off, ent = oracle.invert(p.cu_seqlens, bi, 16)
    boff, bent = _brute_invert(p.cu_seqlens, bi, 16)
    assert np.array_equal(off, boff) and np.array_equal(ent, bent)


def test_invert_round_trip_and_sorted():
    p = ni.make_problem([1000, 513], hq=4, hkv=4, head_dim=8, block_size=64, topk=8, seed=22,
                        with_dout=False)
    off, ent = oracle.invert(p.cu_seqlens, p.block_idx, 64)
    cu = p.cu_seqlens.astype(np.int64)
    T, hkv, topk = p.block_idx.shape
    seq = np.searchsorted(cu, np.arange(T), side="right") - 1
    qb = (np.arange(T) - cu[seq]) // 64
    valid = (p.block_idx >= 0) & (p.block_idx <= qb[:, None, None])
    assert off[-1] == valid.sum() == len(ent)
    nbs = [(int(cu[s + 1] - cu[s]) + 63) // 64 for s in range(len(cu) - 1)]
    blkoff = np.concatenate([[0], np.cumsum(nbs)])
    NB = blkoff[-1]
    got = set()
    for bucket in range(len(off) - 1):
        g, B = divmod(bucket, NB)
        s = np.searchsorted(blkoff, B, side="right") - 1
        lst = ent[off[bucket]:off[bucket + 1]]
        assert (np.diff(lst) > 0).all()                      # ascending in t (then slot)
        for e in lst:
            t, j = divmod(int(e), 64)
            assert p.block_idx[t, g, j] == B - blkoff[s] and seq[t] == s
            got.add((t, g, j))
    want = set(zip(*np.nonzero(valid)))
    assert got == {(int(a), int(b), int(c)) for a, b, c in want}


# ----------------------------------------------------------------------- input recipe pins

def test_inputs_recipe():
    cu = ni.cu_seqlens_from_lengths([1000, 300])
    bi = ni.make_block_idx(cu, 3, 16, 64, seed=4)
    for s in range(2):
        for t in range(int(cu[s]), int(cu[s + 1])):
            qb = (t - int(cu[s])) // 64
            for g in range(3):
                row = bi[t, g]
                vals = row[row >= 0]
                assert len(set(vals.tolist())) == len(vals)
                assert (vals <= qb).all()
                assert row[0] == 0
                if qb >= 1:
                    assert row[1] == qb
                if qb >= 2:
                    assert row[2] == qb - 1
                want = min(16, 1 + min(qb, 1) + (1 if qb >= 2 else 0) + max(qb - 2, 0))
                assert len(vals) == want
                assert (row[len(vals):] == -1).all()
    x = np.array([1.0, 1.00390625, 1.005859375, -2.0e-3, 3.3], dtype=np.float32)
    r = ni.bf16_round(x)
    assert np.array_equal(r, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


# --------------------------------------------------------------------------- sliding window
# window W > 0 keeps, of the selected keys, those with j > i - W (the W most recent
# positions, the query's own included; the module's window_size in the project page's
# quick start).

def _band_sdpa_f64(q, k, v, dout, cu, scale, W):
    """Dense causal attention restricted to a band of W positions, torch float64 with an
    explicit boolean mask (forward, LSE and the autograd backward of sum(dO * O))."""
    T, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    qt = torch.from_numpy(q.astype(np.float64)).requires_grad_()
    kt = torch.from_numpy(k.astype(np.float64)).requires_grad_()
    vt = torch.from_numpy(v.astype(np.float64)).requires_grad_()
    outs, lses, loss = [], [], 0
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        L = b - a
        i = torch.arange(L)
        mask = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - W)
        qs = qt[a:b].permute(1, 0, 2)
        ks = kt[a:b].repeat_interleave(G, 1).permute(1, 0, 2)
        vs = vt[a:b].repeat_interleave(G, 1).permute(1, 0, 2)
        o = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, attn_mask=mask, scale=scale)
        sc = ((qs @ ks.transpose(1, 2)) * scale).masked_fill(~mask, float("-inf"))
        outs.append(o.permute(1, 0, 2))
        lses.append(torch.logsumexp(sc, dim=-1).permute(1, 0))
        loss = loss + (o.permute(1, 0, 2) * torch.from_numpy(dout[a:b].astype(np.float64))).sum()
    loss.backward()
    return (torch.cat(outs).detach().numpy(), torch.cat(lses).detach().numpy(),
            qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy())


@pytest.mark.parametrize("W", [1, 5, 16, 23])
def test_window_dense_selection_matches_band_sdpa(W):
    lengths, hq, hkv, bs = [64, 37, 1], 4, 2, 16
    cu = ni.cu_seqlens_from_lengths(lengths)
    p = ni.make_problem(lengths, hq=hq, hkv=hkv, head_dim=32, block_size=bs, topk=6, seed=61,
                        block_idx=_all_blocks_idx(cu, hkv, bs, 6, np.random.default_rng(7)))
    o, l = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, bs, p.scale, window=W)
    dq, dk, dv = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, bs, p.scale,
                            window=W)
    ro, rl, rdq, rdk, rdv = _band_sdpa_f64(p.q, p.k, p.v, p.dout, cu, p.scale, W)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, rl, rtol=0, atol=1e-12)
    for a, b in ((dq, rdq), (dk, rdk), (dv, rdv)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


def test_window_closed_forms_and_invariance():
    p = ni.make_problem([300, 90], hq=4, hkv=2, head_dim=32, block_size=16, topk=5, seed=62)
    base = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, 16, p.scale)
    wide = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, 16, p.scale, window=300)
    assert np.array_equal(base[0], wide[0]) and np.array_equal(base[1], wide[1])
    gb = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, 16, p.scale)
    gw = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, 16, p.scale, window=300)
    for a, b in zip(gb, gw):   # dK / dV sum over OpenMP threads: equal up to that order
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)
    # W = 1: every query sees only itself (its own block is always selected)
    o, l = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, 16, p.scale, window=1)
    G = 2
    for t in (0, 17, 299, 300, 389):
        for h in range(4):
            kk = p.k[t, h // G].astype(np.float64)
            np.testing.assert_allclose(o[t, h], p.v[t, h // G].astype(np.float64), rtol=0, atol=1e-15)
            assert l[t, h] == pytest.approx(p.scale * float(kk @ p.q[t, h].astype(np.float64)),
                                            rel=0, abs=1e-12)


def test_window_partial_entry_points_match_full():
    p = ni.make_problem([200], hq=4, hkv=1, head_dim=32, block_size=16, topk=6, seed=63)
    W = 40
    dq, dk, dv = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, 16, p.scale,
                            window=W)
    toks = np.array([0, 39, 40, 41, 150, 199])
    np.testing.assert_allclose(
        oracle.bwd_dq(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, 16, p.scale, toks,
                      window=W), dq[toks], rtol=0, atol=1e-13)
    k2, v2 = oracle.bwd_dkdv_keys(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, 16, p.scale,
                                  0, 32, 48, window=W)
    np.testing.assert_allclose(k2, dk[32:80, 0], rtol=0, atol=1e-13)
    np.testing.assert_allclose(v2, dv[32:80, 0], rtol=0, atol=1e-13)
