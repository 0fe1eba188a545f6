"""Parity of threshold-pruned block attention (through the C ABI) with the fp64 BSFA
oracle.  Rows whose block maxima lie within 1e-3 of their threshold are left out of
the comparison: there the fp32 kernel and the fp64 oracle may decide differently."""
import numpy as np
import pytest
import torch

import block_sparse_attention_selected_b200 as nsa
import nsa_inputs as ni
from gpu_util import TOL_LSE, TOL_O, f64, o_gate
from oracle import bsfa

pytestmark = pytest.mark.gpu


def _near_threshold_rows(p, tau, bs=64):
    """(T, hq) mask of rows with a block maximum within 1e-3 of the row's threshold."""
    cu = p.cu_seqlens.astype(np.int64)
    T, hq, _ = p.q.shape
    G = hq // p.k.shape[1]
    near = np.zeros((T, hq), dtype=bool)
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        for h in range(hq):
            S = p.scale * (p.q[a:b, h].astype(np.float64) @ p.k[a:b, h // G].astype(np.float64).T)
            S[np.triu_indices(b - a, 1)] = -np.inf
            for blk in range(0, b - a, bs):
                m = S[:, blk:blk + bs].max(axis=1)
                near[a:b, h] |= np.abs(m - tau[h]) < 1e-3
    return near


@pytest.mark.parametrize("lengths,hq,hkv,taus", [
    ([1000, 77, 0, 300], 8, 2, [-np.inf, 1.5, 2.0, 2.5]),
    ([700], 4, 4, [1.0, 2.2, 2.8, 3.5]),
    ([500, 260], 16, 1, [-np.inf, 2.0, 2.4, 1e9]),
])
def test_bsfa_matches_oracle(lengths, hq, hkv, taus):
    p = ni.make_problem(lengths, hq=hq, hkv=hkv, head_dim=128, block_size=64, topk=4, seed=81,
                        with_dout=False)
    tau = np.resize(np.asarray(taus, dtype=np.float64), hq)
    dev = torch.device("cuda", 0)
    f = lambda a: torch.from_numpy(a).to(dev).to(torch.bfloat16)
    out, lse = nsa.nsa_sel_bsfa_fwd(f(p.q), f(p.k), f(p.v), torch.from_numpy(p.cu_seqlens).to(dev),
                                torch.from_numpy(tau.astype(np.float32)).to(dev), p.scale)
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status() == 0
    ro, rl, _ = bsfa.bsfa_fwd(p.q, p.k, p.v, p.cu_seqlens, 64, p.scale, tau)
    keep = ~_near_threshold_rows(p, tau)
    o, l = f64(out), f64(lse).T
    assert o_gate(o[keep], ro[keep]) <= TOL_O
    fin = keep & np.isfinite(rl)
    assert np.array_equal(np.isneginf(l[keep]), np.isneginf(rl[keep]))
    assert np.abs(l[fin] - rl[fin]).max(initial=0.0) <= TOL_LSE
    assert not o[keep & ~np.isfinite(rl)].any()
