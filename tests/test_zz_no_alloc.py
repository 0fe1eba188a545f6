"""The inversion entry point that allocates nothing.

Some callers cannot allocate device memory themselves (a plug-in inside a framework
that owns all device memory and gives plug-ins no allocation hook, or a loop where
cudaMalloc is not allowed), so nsa_sel_invert_index_noalloc takes its scratch from a
fixed array in the library's own device data.  This file is collected last so that a
run stopping at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_selected_b200 as nsa
import nsa_inputs as ni

pytestmark = pytest.mark.gpu


def _case(lengths, hkv, topk, bs, seed):
    p = ni.make_problem(lengths, hq=hkv, hkv=hkv, head_dim=8, block_size=bs, topk=topk, seed=seed,
                        with_dout=False)
    return torch.from_numpy(p.cu_seqlens).cuda(), torch.from_numpy(p.block_idx).cuda(), bs


def test_noalloc_inversion_matches_workspace_inversion_twice():
    # two calls in a row with different problems: the second must not see the
    # first call's leftovers in the shared scratch array; each result equals the
    # workspace inversion's and, bit for bit, the oracle's
    import oracle
    for lengths, hkv, topk, bs, seed in (([3000, 777, 1], 4, 16, 64, 41), ([5000], 2, 8, 128, 42)):
        cu, bi, bs = _case(lengths, hkv, topk, bs, seed)
        ref_off, ref_ent = nsa.nsa_sel_invert_index(cu, bi, bs)
        off, ent = nsa.nsa_sel_invert_index_noalloc(cu, bi, bs)
        torch.cuda.synchronize()
        assert torch.equal(off, ref_off)
        assert torch.equal(ent, ref_ent)
        o_off, o_ent = oracle.invert(cu.cpu().numpy(), bi.cpu().numpy(), bs)
        assert np.array_equal(off.cpu().numpy(), o_off)
        assert np.array_equal(ent.cpu().numpy(), o_ent)


def test_noalloc_inversion_of_nothing():
    # no tokens: empty lists, and the next call is unaffected
    cu = torch.zeros(2, dtype=torch.int32, device="cuda")
    bi = torch.empty((0, 2, 8), dtype=torch.int32, device="cuda")
    off, ent = nsa.nsa_sel_invert_index_noalloc(cu, bi, 64)
    torch.cuda.synchronize()
    assert ent.numel() == 0 and bool((off == 0).all())
    cu, bi, bs = _case([700], 2, 8, 64, 43)
    off, ent = nsa.nsa_sel_invert_index_noalloc(cu, bi, bs)
    ref_off, ref_ent = nsa.nsa_sel_invert_index(cu, bi, bs)
    torch.cuda.synchronize()
    assert torch.equal(off, ref_off) and torch.equal(ent, ref_ent)


def test_noalloc_rejects_sizes_beyond_the_array():
    lib = nsa.load_library()
    limit = lib.nsa_sel_invert_index_noalloc_max_bytes()
    assert limit == 64 << 20
    P = ctypes.c_void_p
    fake = P(1 << 20)        # never dereferenced: the size check fails first
    # 2^22 tokens x 4 KV heads x 16 slots is inside the supported domain but needs
    # about 4 GB of inversion scratch, far more than the 64 MiB array
    rc = lib.nsa_sel_invert_index_noalloc(fake, 1, 1 << 22, 4, fake, 16, 64, fake, fake, fake,
                                          None)
    assert rc == 3   # NSA_ERR_WORKSPACE
