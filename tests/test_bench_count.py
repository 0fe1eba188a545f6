"""Host-side counting of the benchmark (CPU only): the useful-FLOP key count against a
brute-force restatement of its definition (keys j <= i in a selected block, each
distinct block once; -1, future and out-of-range values select nothing)."""
import numpy as np

import bench
import nsa_inputs as ni


def _brute_keys(cu, bidx, bs):
    T, hkv, _ = bidx.shape
    out = np.zeros((T, hkv), dtype=np.int64)
    for s in range(len(cu) - 1):
        for t in range(int(cu[s]), int(cu[s + 1])):
            i = t - int(cu[s])
            for g in range(hkv):
                sel = {int(b) for b in bidx[t, g] if b >= 0}
                out[t, g] = sum(1 for j in range(i + 1) if j // bs in sel)
    return out


def test_attended_keys_brute_force():
    p = ni.make_problem([300, 77, 0, 5], hq=4, hkv=2, head_dim=8, block_size=16, topk=12, seed=3)
    bi = p.block_idx.copy()
    bi[60, 0, :3] = [2, 2, 40]         # a repeat counts once, an out-of-range value never
    got = bench.attended_keys(p.cu_seqlens, bi, 16)
    assert np.array_equal(got, _brute_keys(p.cu_seqlens, bi, 16))


def test_useful_flops_formula():
    p = ni.make_problem([200], hq=8, hkv=2, head_dim=128, block_size=64, topk=4, seed=4)
    keys = _brute_keys(p.cu_seqlens, p.block_idx, 64)
    fwd, bwd = bench.useful_flops(p)
    assert fwd == 4 * 128 * keys.sum() * 4 and bwd == 2.5 * fwd
