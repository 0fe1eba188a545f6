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
