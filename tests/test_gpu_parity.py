"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small problems are compared element by element over every output; so are the
headline forward and the training shape's forward and backward at their full sizes;
the other full-size workloads are compared on stratified token samples that the
oracle computes one by one.  Tolerances: |O - O_ref| <= 1e-2 on every element whose
exact value has |O_ref| < 2, and beyond half a bf16 ulp of O_ref (the rounding of the
exact answer to the bf16 output) where |O_ref| >= 2; <= 1e-3 on fp32 LSE; relative
Frobenius <= 2e-2 on dQ, dK, dV; the inversion is bit-exact.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_selected_b200 as nsa
import nsa_inputs as ni
import oracle
from gpu_util import (TOL_GRAD, TOL_LSE, TOL_O, f64, max_abs, o_errors, o_gate, rel_fro,
                      sample_tokens, to_device)

pytestmark = pytest.mark.gpu


def _perturb(p: ni.Problem, seed: int, frac: float = 0.05) -> ni.Problem:
    """Shuffle every index row (moving the -1 pads) and plant future, out-of-range and
    negative values in random slots (all must contribute nothing)."""
    rng = np.random.default_rng(seed)
    bi = p.block_idx.copy()
    T, hkv, topk = bi.shape
    idx = np.argsort(rng.random(bi.shape), axis=2)
    bi = np.take_along_axis(bi, idx, axis=2)
    pad = np.argwhere(bi == -1)
    if len(pad):
        pick = pad[rng.random(len(pad)) < frac * 4]
        cu = p.cu_seqlens.astype(np.int64)
        seq = np.searchsorted(cu, pick[:, 0], side="right") - 1
        L = cu[seq + 1] - cu[seq]
        nb = (L + p.block_size - 1) // p.block_size
        kind = rng.integers(0, 3, size=len(pick))
        vals = np.where(kind == 0, nb + 3, np.where(kind == 1, -7, nb - 1))   # oob, negative, last
        bi[pick[:, 0], pick[:, 1], pick[:, 2]] = vals.astype(np.int32)
        # "last block" is a future block for most tokens; keep rows distinct
        for (t, g, _), v in zip(pick, vals):
            row = bi[t, g]
            if (row == v).sum() > 1:
                row[np.nonzero(row == v)[0][1:]] = -1
    p.block_idx = np.ascontiguousarray(bi)
    return p


def _fwd(p):
    d = to_device(p)
    out, lse = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], p.block_size,
                                    p.scale)
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status() == 0
    return d, out, lse


def _check_fwd(p, out, lse, tokens=None):
    o_ref, l_ref = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, p.block_size, p.scale,
                              tokens=tokens)
    o = f64(out) if tokens is None else f64(out[torch.from_numpy(tokens).cuda()])
    l = f64(lse).T if tokens is None else f64(lse[:, torch.from_numpy(tokens).cuda()]).T
    (raw, eo), el = o_errors(o, o_ref), max_abs(l, l_ref)
    assert eo <= TOL_O and el <= TOL_LSE, (p.name, "gated", eo, "raw", raw, "lse", el)
    return eo, el


# ------------------------------------------------------------------------- inversion

INV_CASES = [
    ("tiny", dict(lengths=[2048], hq=4, hkv=4, block_size=64, topk=8, seed=1), False),
    ("varlen_ragged", dict(lengths=[700, 37, 1, 515], hq=2, hkv=2, block_size=64, topk=16, seed=3), True),
    ("bs128_k64", dict(lengths=[3000, 129], hq=4, hkv=1, block_size=128, topk=64, seed=5), True),
    ("empty_seq", dict(lengths=[0, 300, 0, 65], hq=3, hkv=3, block_size=64, topk=5, seed=6), True),
    # many short sequences, empty ones among them: a sort thread's entries cross several
    # sequence boundaries
    ("many_seqs", dict(lengths=[int(x) for x in np.random.default_rng(7).integers(0, 90, 160)],
                       hq=4, hkv=2, block_size=64, topk=3, seed=7), True),
]


@pytest.mark.parametrize("name,spec,perturb", INV_CASES, ids=[c[0] for c in INV_CASES])
def test_invert_bit_exact_small(name, spec, perturb):
    p = ni.make_problem(head_dim=8, with_dout=False, **spec)
    if perturb:
        p = _perturb(p, 11)
    cu = torch.from_numpy(p.cu_seqlens).cuda()
    bi = torch.from_numpy(p.block_idx).cuda()
    off, ent = nsa.nsa_sel_invert_index(cu, bi, p.block_size)
    roff, rent = oracle.invert(p.cu_seqlens, p.block_idx, p.block_size)
    assert np.array_equal(off.cpu().numpy(), roff)
    assert np.array_equal(ent.cpu().numpy(), rent)


@pytest.mark.parametrize("wl", [ni.HEADLINE, "varlen_64k_32k_g1_k16", "train_t32k_hq64_g8_k16",
                                "sweep_t64k_g1_bs128_k32"])
def test_invert_bit_exact_full(wl):
    spec = ni.WORKLOADS[wl]
    cu = ni.cu_seqlens_from_lengths(spec["lengths"])
    bidx = ni.make_block_idx(cu, spec["hkv"], spec["topk"], spec["block_size"], spec["seed"])
    off, ent = nsa.nsa_sel_invert_index(torch.from_numpy(cu).cuda(), torch.from_numpy(bidx).cuda(),
                                        spec["block_size"])
    roff, rent = oracle.invert(cu, bidx, spec["block_size"])
    assert np.array_equal(off.cpu().numpy(), roff)
    assert np.array_equal(ent.cpu().numpy(), rent)


# --------------------------------------------------------------------------- forward

FWD_SMALL = [
    ("tiny_t2k_g1_k8", None, False),
    ("g1_bs64_k16", dict(lengths=[700, 37, 1, 515], hq=2, hkv=2, block_size=64, topk=16, seed=7), True),
    ("g2_bs64_k3", dict(lengths=[1500, 130], hq=4, hkv=2, block_size=64, topk=3, seed=8), True),
    ("g4_bs64_k16", dict(lengths=[2500, 64, 63], hq=8, hkv=2, block_size=64, topk=16, seed=9), True),
    ("g8_bs128_k8", dict(lengths=[2000, 1], hq=16, hkv=2, block_size=128, topk=8, seed=10), True),
    ("g16_bs128_k64", dict(lengths=[1800], hq=16, hkv=1, block_size=128, topk=64, seed=11), True),
    ("g16_bs64_k1", dict(lengths=[999, 333], hq=32, hkv=2, block_size=64, topk=1, seed=12), False),
    ("g4_dense_causal", dict(lengths=[640, 300], hq=8, hkv=2, block_size=64, topk=12, seed=13), False),
    ("g32_bs64_k8", dict(lengths=[600, 77], hq=64, hkv=2, block_size=64, topk=8, seed=14), True),
    ("g128_bs128_k4", dict(lengths=[300], hq=128, hkv=1, block_size=128, topk=4, seed=15), False),
]


@pytest.mark.parametrize("name,spec,perturb", FWD_SMALL, ids=[c[0] for c in FWD_SMALL])
def test_fwd_small_full_compare(name, spec, perturb):
    if spec is None:
        p = ni.workload(name, with_dout=False)
    else:
        p = ni.make_problem(name=name, with_dout=False, **spec)
    if name == "g4_dense_causal":   # topk covers every block: dense causal attention
        cu = p.cu_seqlens.astype(np.int64)
        for s in range(p.nseq):
            L = int(cu[s + 1] - cu[s])
            nb = (L + 63) // 64
            p.block_idx[cu[s]:cu[s + 1]] = -1
            p.block_idx[cu[s]:cu[s + 1], :, :nb] = np.arange(nb, dtype=np.int32)[::-1]
    if perturb:
        p = _perturb(p, 5)
    _, out, lse = _fwd(p)
    _check_fwd(p, out, lse)


# Every point of the T=65536 sweep (group 1-16, block 64 / 128, topk 8 / 16 / 32).
FWD_FULL = ["fwd_t32k_hq32_g4_k16", "varlen_64k_32k_g1_k16", "train_t32k_hq64_g8_k16"] + \
    [f"sweep_t64k_g{g}_bs{bs}_k{k}" for g, bs, k in ni.SWEEP_POINTS]
# Compared on every output element (the oracle needs up to ~30 s for each on 16 cores);
# the other sweep points on stratified token samples.
FWD_FULL_EVERY_ELEMENT = {ni.HEADLINE, "fwd_t32k_hq32_g4_k16", "varlen_64k_32k_g1_k16",
                          "train_t32k_hq64_g8_k16"}


@pytest.mark.parametrize("bs", [64, 128])
def test_fwd_large_v_uses_block_exponent(bs):
    """V scaled by 2^15 (exact in bf16): |V| reaches ~1.6e5, above fp16's range, so the
    forward must carry the per-block exponent e > 0 through its fp16 partials."""
    p = ni.make_problem([1500, 300], hq=8, hkv=2, block_size=bs, topk=8, seed=41,
                        name=f"large_v_bs{bs}")
    p.v = (p.v * 32768.0).astype(p.v.dtype)
    assert np.abs(p.v).max() > 65504.0
    _, out, lse = _fwd(p)
    assert torch.isfinite(out.float()).all()
    # O scales exactly with V (a power of two), LSE does not change: compare O / 2^15
    # with the standard tolerance (bf16 rounding is invariant under that scaling)
    o_ref, l_ref = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, p.block_size, p.scale)
    eo = o_gate(f64(out) / 32768.0, o_ref / 32768.0)
    el = max_abs(f64(lse).T, l_ref)
    assert eo <= TOL_O and el <= TOL_LSE, (p.name, eo, el)


@pytest.mark.parametrize("wl", FWD_FULL)
def test_fwd_full_size(wl):
    p = ni.workload(wl, with_dout=False)
    _, out, lse = _fwd(p)
    if wl in FWD_FULL_EVERY_ELEMENT:
        _check_fwd(p, out, lse)
    else:
        toks = sample_tokens(p.cu_seqlens, p.block_size, n_random=96, seed=1)
        _check_fwd(p, out, lse, tokens=toks)
    # properties that hold on every element at any size: finite outputs
    assert torch.isfinite(out.float()).all()
    assert torch.isfinite(lse).all()


def test_fwd_deterministic_and_zero_tokens():
    p = ni.make_problem([1200, 77], hq=8, hkv=2, block_size=64, topk=16, seed=21, with_dout=False)
    d, o1, l1 = _fwd(p)
    o2, l2 = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], 64, p.scale)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # T = 0: a no-op that still succeeds
    z = torch.empty((0, 8, 128), dtype=torch.bfloat16, device="cuda")
    zk = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(2, dtype=torch.int32, device="cuda")
    bi = torch.empty((0, 2, 16), dtype=torch.int32, device="cuda")
    o, l = nsa.nsa_sel_attn_fwd(z, zk, zk, cu, bi, 64)
    assert o.shape == (0, 8, 128) and l.shape == (8, 0)


def test_fwd_empty_rows_give_zero_and_neg_inf():
    p = ni.make_problem([500], hq=4, hkv=2, block_size=64, topk=4, seed=22, with_dout=False)
    p.block_idx[100, 0] = -1
    p.block_idx[200, 1] = [-1, 9, -4, 8]        # only out-of-range / future values
    _, out, lse = _fwd(p)
    assert (out[100, 0:2].float() == 0).all() and torch.isneginf(lse[0:2, 100]).all()
    assert (out[200, 2:4].float() == 0).all() and torch.isneginf(lse[2:4, 200]).all()
    _check_fwd(p, out, lse)


def test_bad_cu_seqlens_reported():
    p = ni.make_problem([256, 256], hq=2, hkv=2, block_size=64, topk=4, seed=23, with_dout=False)
    d = to_device(p)
    cu = torch.tensor([0, 300, 200], dtype=torch.int32, device="cuda")   # decreasing, wrong end
    nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], cu, d["bidx"], 64)
    assert nsa.nsa_sel_check_status() == 6


def test_validate_indices_counts():
    p = ni.make_problem([300, 100], hq=2, hkv=2, block_size=64, topk=6, seed=24, with_dout=False)
    bi = p.block_idx.copy()
    bi[10, 0, 5] = 99        # out of range
    bi[150, 1, 4] = -3       # out of range
    bi[299, 1, 5] = bi[299, 1, 0]   # duplicate
    d_cu = torch.from_numpy(p.cu_seqlens).cuda()
    assert nsa.nsa_sel_validate_indices(d_cu, torch.from_numpy(p.block_idx).cuda(), 64) == (0, 0)
    assert nsa.nsa_sel_validate_indices(d_cu, torch.from_numpy(bi).cuda(), 64) == (2, 1)


# -------------------------------------------------------------------------- backward

def _bwd(p, d, out, lse):
    dq, dk, dv = nsa.nsa_sel_attn_bwd(d["q"], d["k"], d["v"], out, lse, d["dout"], d["cu"],
                                      d["bidx"], p.block_size, p.scale)
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status() == 0
    return dq, dk, dv


BWD_SMALL = [
    ("tiny_t2k_g1_k8", None, False),
    ("g4_bs64_k16", dict(lengths=[1500, 40, 300], hq=8, hkv=2, block_size=64, topk=16, seed=31), True),
    ("g1_bs128_k8", dict(lengths=[1100, 1], hq=2, hkv=2, block_size=128, topk=8, seed=32), True),
    ("g16_bs64_k5", dict(lengths=[700], hq=16, hkv=1, block_size=64, topk=5, seed=33), False),
    ("g8_bs128_k64", dict(lengths=[900, 129], hq=8, hkv=1, block_size=128, topk=64, seed=34), True),
    ("g32_bs64_k6", dict(lengths=[500, 70], hq=32, hkv=1, block_size=64, topk=6, seed=35), True),
    ("g128_bs64_k3", dict(lengths=[260], hq=128, hkv=1, block_size=64, topk=3, seed=37), False),
]


@pytest.mark.parametrize("name,spec,perturb", BWD_SMALL, ids=[c[0] for c in BWD_SMALL])
def test_bwd_small_full_compare(name, spec, perturb):
    p = ni.workload(name) if spec is None else ni.make_problem(name=name, **spec)
    if perturb:
        p = _perturb(p, 6)
    d, out, lse = _fwd(p)
    dq, dk, dv = _bwd(p, d, out, lse)
    rdq, rdk, rdv = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, p.block_size,
                               p.scale)
    e = (rel_fro(f64(dq), rdq), rel_fro(f64(dk), rdk), rel_fro(f64(dv), rdv))
    assert max(e) <= TOL_GRAD, (name, e)


def _check_bwd_sampled(p, dq, dk, dv, blocks, seed=0, n_random=48):
    toks = sample_tokens(p.cu_seqlens, p.block_size, n_random=n_random, seed=seed)
    rdq = oracle.bwd_dq(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, p.block_size, p.scale,
                        toks)
    e_dq = rel_fro(f64(dq[torch.from_numpy(toks).cuda()]), rdq)
    gk, rk, gv, rv = [], [], [], []
    for g, key0, n in blocks:
        k_ref, v_ref = oracle.bwd_dkdv_keys(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx,
                                            p.block_size, p.scale, g, key0, n)
        gk.append(f64(dk[key0:key0 + n, g]))
        gv.append(f64(dv[key0:key0 + n, g]))
        rk.append(k_ref)
        rv.append(v_ref)
    e_dk = rel_fro(np.concatenate(gk), np.concatenate(rk))
    e_dv = rel_fro(np.concatenate(gv), np.concatenate(rv))
    assert max(e_dq, e_dk, e_dv) <= TOL_GRAD, (p.name, e_dq, e_dk, e_dv)


def test_bwd_medium_multi_unit():
    """Block 0 is selected by every token: 512 tiles, 16 backward work units."""
    p = ni.make_problem([8192], hq=16, hkv=2, block_size=64, topk=16, seed=35, name="bwd_medium")
    d, out, lse = _fwd(p)
    dq, dk, dv = _bwd(p, d, out, lse)
    _check_bwd_sampled(p, dq, dk, dv, blocks=[(0, 0, 64), (1, 64, 64), (1, 4096, 64),
                                              (0, 8128, 64)])


def test_bwd_full_size_training_shape():
    """The training shape (T = 32768, 64 query heads, 8 KV heads, topk 16): dQ, dK and dV
    compared with the oracle over the whole tensors (about 100 s of oracle time on 16
    cores), block 0 -- selected by every token -- included."""
    p = ni.workload("train_t32k_hq64_g8_k16")
    d, out, lse = _fwd(p)
    dq, dk, dv = _bwd(p, d, out, lse)
    assert torch.isfinite(dq.float()).all() and torch.isfinite(dk.float()).all()
    assert torch.isfinite(dv.float()).all()
    rdq, rdk, rdv = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, p.block_size,
                               p.scale)
    e = (rel_fro(f64(dq), rdq), rel_fro(f64(dk), rdk), rel_fro(f64(dv), rdv))
    # block 0 of every KV head on its own (the most-reduced keys)
    e0 = max(rel_fro(f64(dk[:64]), rdk[:64]), rel_fro(f64(dv[:64]), rdv[:64]))
    assert max(e) <= TOL_GRAD and e0 <= TOL_GRAD, (e, e0)


def test_bwd_deterministic():
    p = ni.make_problem([3000], hq=8, hkv=2, block_size=64, topk=16, seed=36)
    d, out, lse = _fwd(p)
    a = _bwd(p, d, out, lse)
    b = _bwd(p, d, out, lse)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_repeat_calls_bitwise_identical():
    # many back-to-back calls at a size with a few hundred tiles per SM: every one must
    # reproduce the first bit for bit (a hazard between pipelined hand-offs would show as
    # an occasional difference in a few rows)
    p = ni.make_problem([16384], hq=16, hkv=4, block_size=64, topk=16, seed=41)
    d, out0, lse0 = _fwd(p)
    for _ in range(100):
        o, l = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], 64, p.scale)
        assert torch.equal(o, out0) and torch.equal(l, lse0)
    g0 = _bwd(p, d, out0, lse0)
    for _ in range(30):
        for x, y in zip(_bwd(p, d, out0, lse0), g0):
            assert torch.equal(x, y)


def test_bwd_reusing_forward_inversion():
    p = ni.make_problem([2500, 700], hq=8, hkv=2, block_size=64, topk=16, seed=42)
    d = to_device(p)
    T, hq, hkv, topk = p.q.shape[0], p.q.shape[1], p.k.shape[1], p.block_idx.shape[2]
    nb = nsa.nsa_sel_attn_workspace_size(T, 2, hq, hkv, 128, topk, 64, True)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    out, lse = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], 64, p.scale,
                                    workspace=ws)
    ref = nsa.nsa_sel_attn_bwd(d["q"], d["k"], d["v"], out, lse, d["dout"], d["cu"], d["bidx"],
                               64, p.scale)
    got = nsa.nsa_sel_attn_bwd(d["q"], d["k"], d["v"], out, lse, d["dout"], d["cu"], d["bidx"],
                               64, p.scale, workspace=ws, reuse_index=True)
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status(ws) == 0
    for x, y in zip(got, ref):
        assert torch.equal(x, y)
    # an inversion of other index tensors is refused (device status), not used
    bidx2 = d["bidx"].clone()
    nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], bidx2, 64, p.scale, workspace=ws)
    nsa.nsa_sel_attn_bwd(d["q"], d["k"], d["v"], out, lse, d["dout"], d["cu"], d["bidx"], 64,
                         p.scale, workspace=ws, reuse_index=True)
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status(ws) == 1   # NSA_ERR_INVALID_ARG


def test_fwd_without_lse():
    # a forward with no backward: null LSE, the same output
    p = ni.make_problem([900, 300], hq=8, hkv=2, block_size=64, topk=8, seed=43, with_dout=False)
    d, out, _ = _fwd(p)
    o2, l2 = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], 64, p.scale,
                                  with_lse=False)
    torch.cuda.synchronize()
    assert l2 is None and torch.equal(o2, out)
    assert nsa.nsa_sel_check_status() == 0


FP16_CASES = [
    ("f16_g4_bs64_k16", dict(lengths=[1500, 300], hq=8, hkv=2, block_size=64, topk=16, seed=51), True),
    ("f16_g2_bs128_k8", dict(lengths=[900, 65], hq=4, hkv=2, block_size=128, topk=8, seed=52), False),
]


@pytest.mark.parametrize("name,spec,perturb", FP16_CASES, ids=[c[0] for c in FP16_CASES])
def test_fp16_fwd_bwd_full_compare(name, spec, perturb):
    # fp16 attention tensors: the generator's values rounded to fp16, and the oracle
    # given exactly those values
    p = ni.make_problem(name=name, **spec)
    if perturb:
        p = _perturb(p, 7)
    for a in ("q", "k", "v", "dout"):
        setattr(p, a, getattr(p, a).astype(np.float16).astype(np.float32))
    d = to_device(p, dtype=torch.float16)
    out, lse = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], p.block_size,
                                    p.scale)
    dq, dk, dv = nsa.nsa_sel_attn_bwd(d["q"], d["k"], d["v"], out, lse, d["dout"], d["cu"],
                                      d["bidx"], p.block_size, p.scale)
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status() == 0
    assert out.dtype == dq.dtype == dk.dtype == dv.dtype == torch.float16
    _check_fwd(p, out, lse)
    rdq, rdk, rdv = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, p.block_size,
                               p.scale)
    e = (rel_fro(f64(dq), rdq), rel_fro(f64(dk), rdk), rel_fro(f64(dv), rdv))
    assert max(e) <= TOL_GRAD, (name, e)


# ------------------------------------------------------------------ sliding window

WINDOW_CASES = [
    # name, problem, window, perturb
    ("w512_g4_bs64_k16", dict(lengths=[1500, 40, 700], hq=8, hkv=2, block_size=64, topk=16, seed=61), 512, True),
    ("w100_g1_bs128_k8", dict(lengths=[1100, 1], hq=2, hkv=2, block_size=128, topk=8, seed=62), 100, True),
    ("w1_g16_bs64_k5", dict(lengths=[700], hq=16, hkv=1, block_size=64, topk=5, seed=63), 1, False),
    ("w70_g8_bs64_k12", dict(lengths=[900, 129], hq=8, hkv=1, block_size=64, topk=12, seed=64), 70, True),
]


@pytest.mark.parametrize("name,spec,W,perturb", WINDOW_CASES, ids=[c[0] for c in WINDOW_CASES])
def test_window_fwd_bwd_full_compare(name, spec, W, perturb):
    # selection and a sliding window of W keys; some rows keep no key (O = 0, LSE = -inf)
    p = ni.make_problem(name=name, **spec)
    if perturb:
        p = _perturb(p, 8)
    d = to_device(p)
    out, lse = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], p.block_size,
                                    p.scale, window_size=W)
    dq, dk, dv = nsa.nsa_sel_attn_bwd(d["q"], d["k"], d["v"], out, lse, d["dout"], d["cu"],
                                      d["bidx"], p.block_size, p.scale, window_size=W)
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status() == 0
    o_ref, l_ref = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, p.block_size, p.scale,
                              window=W)
    o, l = f64(out), f64(lse).T
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(l), fin), name
    assert not o[~fin].any(), name
    eo, el = o_gate(o, o_ref), max_abs(l[fin], l_ref[fin])
    assert eo <= TOL_O and el <= TOL_LSE, (name, eo, el)
    rdq, rdk, rdv = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, p.block_size,
                               p.scale, window=W)
    e = (rel_fro(f64(dq), rdq), rel_fro(f64(dk), rdk), rel_fro(f64(dv), rdv))
    assert max(e) <= TOL_GRAD, (name, e)


@pytest.mark.parametrize("bs,W", [(64, 512), (128, 300)])
def test_window_sliding_branch_is_band_attention(bs, W):
    # the sliding branch: every block the window reaches selected -> banded causal attention
    p = ni.make_problem([2100, 333], hq=8, hkv=2, block_size=bs, topk=16, seed=65)
    p.block_idx = ni.band_block_idx(p.cu_seqlens, p.hkv, p.topk, bs, W)
    d = to_device(p)
    out, lse = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], bs, p.scale,
                                    window_size=W)
    dq, dk, dv = nsa.nsa_sel_attn_bwd(d["q"], d["k"], d["v"], out, lse, d["dout"], d["cu"],
                                      d["bidx"], bs, p.scale, window_size=W)
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status() == 0
    _check_fwd_window(p, out, lse, W)
    rdq, rdk, rdv = oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, bs, p.scale,
                               window=W)
    e = (rel_fro(f64(dq), rdq), rel_fro(f64(dk), rdk), rel_fro(f64(dv), rdv))
    assert max(e) <= TOL_GRAD, e


def _check_fwd_window(p, out, lse, W):
    o_ref, l_ref = oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, p.block_size, p.scale,
                              window=W)
    eo, el = o_gate(f64(out), o_ref), max_abs(f64(lse).T, l_ref)
    assert eo <= TOL_O and el <= TOL_LSE, (p.name, eo, el)


def test_window_wider_than_sequences_changes_nothing_and_tags_reuse():
    p = ni.make_problem([1200, 300], hq=8, hkv=2, block_size=64, topk=16, seed=66)
    d = to_device(p)
    T, hq, hkv, topk = p.q.shape[0], p.q.shape[1], p.k.shape[1], p.block_idx.shape[2]
    ref_o, ref_l = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], 64, p.scale)
    nb = nsa.nsa_sel_attn_workspace_size(T, 2, hq, hkv, 128, topk, 64, True)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    o, l = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], 64, p.scale,
                                workspace=ws, window_size=1 << 20)
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status(ws) == 0
    assert torch.equal(o, ref_o) and torch.equal(l, ref_l)
    # the inversion was made for window 1 << 20: a backward with another window refuses it
    nsa.nsa_sel_attn_bwd(d["q"], d["k"], d["v"], o, l, d["dout"], d["cu"], d["bidx"], 64,
                         p.scale, workspace=ws, reuse_index=True, window_size=512)
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status(ws) == 1   # NSA_ERR_INVALID_ARG
