"""Parity of the selection-step kernels (through the C ABI) with the fp64 oracle:
the compressed K / V against ``oracle.selection.compress_kv`` (bf16 rounding of the
exact mean), cu_cmp and the top-k bit-exact against ``select_topk``."""
import numpy as np
import pytest
import torch

import block_sparse_attention_selected_b200 as nsa
import nsa_inputs as ni
from oracle import selection as sel

pytestmark = pytest.mark.gpu


def _half_ulp_bf16(x):
    mag = np.abs(x)
    return np.where(mag > 0, np.exp2(np.floor(np.log2(np.where(mag > 0, mag, 1.0))) - 8), 0.0)


@pytest.mark.parametrize("lengths,hkv", [([2048], 4), ([700, 31, 0, 32, 515, 48], 2),
                                         ([65536], 4)])
def test_compress_kv_matches_oracle(lengths, hkv):
    p = ni.make_problem(lengths, hq=hkv, hkv=hkv, head_dim=128, block_size=64, topk=4, seed=71,
                        with_dout=False)
    dev = torch.device("cuda", 0)
    k = torch.from_numpy(p.k).to(dev).to(torch.bfloat16)
    v = torch.from_numpy(p.v).to(dev).to(torch.bfloat16)
    cu = torch.from_numpy(p.cu_seqlens).to(dev)
    kc, vc, cu_cmp = nsa.nsa_sel_compress_kv(k, v, cu, 32, 16)
    torch.cuda.synchronize()
    rk, rv, rcu = sel.compress_kv(p.k, p.v, p.cu_seqlens, 32, 16)
    assert np.array_equal(cu_cmp.cpu().numpy(), rcu.astype(np.int32))
    n = int(rcu[-1])
    gk = kc[:n].float().cpu().numpy().astype(np.float64)
    gv = vc[:n].float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(gk - rk) <= _half_ulp_bf16(rk) + 1e-6)
    assert np.all(np.abs(gv - rv) <= _half_ulp_bf16(rv) + 1e-6)


def _scores(cu, hkv, nb_stride, seed):
    rng = np.random.default_rng(seed)
    T = int(cu[-1])
    x = rng.random((T, hkv, nb_stride)).astype(np.float32)
    x[:, :, ::3] = np.round(x[:, :, ::3], 1)          # ties
    return x


@pytest.mark.parametrize("lengths,hkv,bs,topk,init,local", [
    ([3000, 1, 640, 0, 129], 2, 64, 16, 1, 2),
    ([2100], 3, 128, 5, 1, 2),
    ([1500, 77], 1, 64, 3, 2, 3),
    ([4096], 2, 64, 64, 1, 2),
])
def test_select_topk_matches_oracle(lengths, hkv, bs, topk, init, local):
    cu = ni.cu_seqlens_from_lengths(lengths)
    nb_stride = max((L + bs - 1) // bs for L in lengths)
    x = _scores(cu, hkv, nb_stride, 72)
    dev = torch.device("cuda", 0)
    got = nsa.nsa_sel_select_topk(torch.from_numpy(x).to(dev), torch.from_numpy(cu).to(dev), bs,
                                  topk, init, local)
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status() == 0
    per_seq = []
    for s in range(len(lengths)):
        a, b = int(cu[s]), int(cu[s + 1])
        per_seq.append(x[a:b].astype(np.float64))
    want = sel.select_topk(per_seq, cu, topk, bs, init, local)
    assert np.array_equal(got.cpu().numpy(), want)


def test_select_topk_full_size_sampled():
    # T = 65536, four KV heads, 1024 blocks of 64: sampled rows against numpy's sort
    cu = ni.cu_seqlens_from_lengths([65536])
    x = _scores(cu, 4, 1024, 73)
    dev = torch.device("cuda", 0)
    got = nsa.nsa_sel_select_topk(torch.from_numpy(x).to(dev), torch.from_numpy(cu).to(dev), 64,
                                  16, 1, 2).cpu().numpy()
    assert nsa.nsa_sel_check_status() == 0
    rng = np.random.default_rng(9)
    for t in np.concatenate([rng.integers(0, 65536, 300), [0, 63, 64, 127, 128, 65535]]):
        qb = int(t) // 64
        for g in range(4):
            forced = [0] + [b for b in (qb, qb - 1) if b > 0]
            forced = list(dict.fromkeys(b for b in forced if b <= qb))[:16]
            free = np.array([b for b in range(qb + 1) if b not in forced], dtype=np.int64)
            order = free[np.lexsort((free, -x[t, g, free].astype(np.float64)))] if len(free) else free
            row = forced + [int(b) for b in order[:16 - len(forced)]]
            want = np.full(16, -1, dtype=np.int32)
            want[:len(row)] = row
            assert np.array_equal(got[t, g], want), (t, g)


def test_select_topk_short_score_rows_reported():
    cu = ni.cu_seqlens_from_lengths([300])
    x = _scores(cu, 1, 3, 74)                         # blocks 0..2 only; token 299 has qb 4
    dev = torch.device("cuda", 0)
    got = nsa.nsa_sel_select_topk(torch.from_numpy(x).to(dev), torch.from_numpy(cu).to(dev), 64,
                                  4, 1, 2)
    assert nsa.nsa_sel_check_status() == 1            # NSA_ERR_INVALID_ARG
    assert np.all(got[299].cpu().numpy() == -1)


def _oracle_scores(p, hkv, bs):
    """Oracle block scores from the oracle's own compressed keys rounded to bf16 (the
    kernel's compressed keys are bf16)."""
    kc, vc, cuc = sel.compress_kv(p.k, p.v, p.cu_seqlens, 32, 16)
    kc = ni.bf16_round(kc.astype(np.float32)).astype(np.float64)
    _, _, probs = sel.compressed_attention(p.q, kc, vc, p.cu_seqlens, cuc, p.scale, 32, 16)
    return sel.block_scores(probs, p.cu_seqlens, hkv, bs, 32, 16)


@pytest.mark.parametrize("lengths,hq,hkv,bs", [([1500, 40, 0, 700], 8, 2, 64),
                                               ([2100], 4, 4, 128),
                                               ([900, 1300], 16, 1, 64),
                                               ([3000], 32, 1, 64)])
def test_block_scores_match_oracle(lengths, hq, hkv, bs):
    p = ni.make_problem(lengths, hq=hq, hkv=hkv, head_dim=128, block_size=bs, topk=4, seed=75,
                        with_dout=False)
    dev = torch.device("cuda", 0)
    f = lambda a: torch.from_numpy(a).to(dev).to(torch.bfloat16)
    q, k, v = f(p.q), f(p.k), f(p.v)
    cu = torch.from_numpy(p.cu_seqlens).to(dev)
    kc, _, cu_cmp = nsa.nsa_sel_compress_kv(k, v, cu)
    nb = max((L + bs - 1) // bs for L in lengths)
    got = nsa.nsa_sel_block_scores(q, kc, cu, cu_cmp, bs, nb, p.scale).cpu().numpy()
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status() == 0
    want = _oracle_scores(p, hkv, bs)
    G = hq // hkv
    for s, ref in enumerate(want):
        a = int(p.cu_seqlens[s])
        for i in range(ref.shape[0]):
            qb = i // bs
            g_ = got[a + i, :, :qb + 1].astype(np.float64)
            assert np.all(np.abs(g_ - ref[i, :, :qb + 1]) <= 1e-3 * G + 1e-3 * np.abs(ref[i, :, :qb + 1])), (s, i)


def test_select_blocks_end_to_end():
    # compression, scores and top-k on the GPU: forced slots exact; every other chosen
    # block scores (by the oracle) within tolerance of the oracle's k-th best
    bs, topk, hkv = 64, 8, 2
    p = ni.make_problem([2500, 600], hq=8, hkv=hkv, head_dim=128, block_size=bs, topk=topk,
                        seed=76, with_dout=False)
    dev = torch.device("cuda", 0)
    f = lambda a: torch.from_numpy(a).to(dev).to(torch.bfloat16)
    bi = nsa.nsa_sel_select_blocks(f(p.q), f(p.k), f(p.v), torch.from_numpy(p.cu_seqlens).to(dev),
                                   bs, topk, 1, 2, max_seqlen=2500, scale=p.scale).cpu().numpy()
    assert nsa.nsa_sel_check_status() == 0
    ref = _oracle_scores(p, hkv, bs)
    want = sel.select_topk(ref, p.cu_seqlens, topk, bs, 1, 2)
    G = 4
    for s in range(2):
        a, L = int(p.cu_seqlens[s]), int(p.cu_seqlens[s + 1] - p.cu_seqlens[s])
        for i in range(L):
            qb = i // bs
            nforced = min(3, qb + 1)
            for g in range(hkv):
                assert np.array_equal(bi[a + i, g, :nforced], want[a + i, g, :nforced])
                row = [int(b) for b in bi[a + i, g] if b >= 0]
                assert len(row) == len(set(row)) == min(topk, qb + 1)
                rest = [int(b) for b in want[a + i, g, nforced:] if b >= 0]
                if rest:
                    kth = ref[s][i, g, rest[-1]]
                    for b in row[nforced:]:
                        assert ref[s][i, g, b] >= kth - 2e-3 * G, (s, i, g, b)
