"""Host-side counting of the benchmark (CPU only): the useful-FLOP key count (with and
without a sliding window) and the sliding branch's index, each against a brute-force
restatement of its definition (keys j <= i, and j > i - W under a window, in a
selected block, each distinct block once; -1, future and out-of-range values select
nothing)."""
import numpy as np
import pytest

import bench
import nsa_inputs as ni


def _brute_keys(cu, bidx, bs, W=0):
    T, hkv, _ = bidx.shape
    out = np.zeros((T, hkv), dtype=np.int64)
    for s in range(len(cu) - 1):
        for t in range(int(cu[s]), int(cu[s + 1])):
            i = t - int(cu[s])
            for g in range(hkv):
                sel = {int(b) for b in bidx[t, g] if b >= 0}
                out[t, g] = sum(1 for j in range(i + 1) if j // bs in sel and (W <= 0 or j > i - W))
    return out


@pytest.mark.parametrize("W", [0, 1, 7, 16, 40, 1 << 20])
def test_attended_keys_brute_force(W):
    p = ni.make_problem([300, 77, 0, 5], hq=4, hkv=2, head_dim=8, block_size=16, topk=12, seed=3)
    bi = p.block_idx.copy()
    bi[60, 0, :3] = [2, 2, 40]         # a repeat counts once, an out-of-range value never
    got = bench.attended_keys(p.cu_seqlens, bi, 16, W)
    assert np.array_equal(got, _brute_keys(p.cu_seqlens, bi, 16, W))


def test_useful_flops_formula():
    p = ni.make_problem([200], hq=8, hkv=2, head_dim=128, block_size=64, topk=4, seed=4)
    keys = _brute_keys(p.cu_seqlens, p.block_idx, 64)
    fwd, bwd = bench.useful_flops(p)
    assert fwd == 4 * 128 * keys.sum() * 4 and bwd == 2.5 * fwd


@pytest.mark.parametrize("bs,W", [(16, 50), (16, 16), (32, 1)])
def test_band_index_reaches_exactly_the_window(bs, W):
    cu = ni.cu_seqlens_from_lengths([200, 0, 33])
    bi = ni.band_block_idx(cu, 2, 8, bs, W)
    for s in range(len(cu) - 1):
        for t in range(int(cu[s]), int(cu[s + 1])):
            i = t - int(cu[s])
            want = {j // bs for j in range(max(0, i - W + 1), i + 1)}
            row = [int(b) for b in bi[t, 0] if b >= 0]
            assert len(row) == len(set(row))
            # every block the window reaches, plus at most one block before it
            assert want <= set(row) and len(set(row) - want) <= 1
            assert np.array_equal(bi[t, 0], bi[t, 1])
    # with the window, the band selects exactly the window's keys
    keys = bench.attended_keys(cu, bi, bs, W)
    i = np.concatenate([np.arange(int(cu[s + 1] - cu[s])) for s in range(len(cu) - 1)])
    assert np.array_equal(keys[:, 0], np.minimum(i + 1, W))
