"""Failure detection on the device, made without faulting the GPU.

Every spin-wait of the kernels is bounded.  The test-only option NSA_TEST_SKIP_ARRIVE
withholds one producer arrival on a barrier that gates no copy or tensor-core work
already in flight, and NSA_TEST_SHORT_WAITS shortens the budget of every bounded
wait to about 8.6 ms: the forward must then report NSA_ERR_TIMEOUT through the
status block, leave its outputs untouched, and the next ordinary call must be exact.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_selected_b200 as nsa
import nsa_inputs as ni
from gpu_util import to_device

pytestmark = pytest.mark.gpu

NSA_ERR_TIMEOUT = 5
NSA_TEST_SHORT_WAITS = 0x100
NSA_TEST_SKIP_ARRIVE = 0x200


def _fwd_ex(d, p, out, lse, ws, flags):
    lib = nsa.load_library()
    T, hq, hkv, topk = p.T, p.hq, p.hkv, p.topk
    sp = nsa._ptr
    with torch.cuda.device(out.device):
        return lib.nsa_sel_attn_fwd_ex(
            sp(d["q"]), sp(d["k"]), sp(d["v"]), sp(d["cu"]), p.nseq, T, hq, hkv, 128, sp(d["bidx"]),
            topk, p.block_size, p.scale, sp(out), sp(lse), sp(ws), ws.numel(),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), flags, 0, None, 0, None)


def test_expired_wait_reports_timeout_and_the_device_stays_usable():
    p = ni.make_problem([3000, 500], hq=8, hkv=2, block_size=64, topk=16, seed=91, with_dout=False)
    d = to_device(p)
    ws = torch.empty(nsa.nsa_sel_attn_workspace_size(p.T, p.nseq, p.hq, p.hkv, 128, p.topk, 64),
                     dtype=torch.uint8, device="cuda")
    ref_o = torch.empty_like(d["q"])
    ref_l = torch.empty((p.hq, p.T), dtype=torch.float32, device="cuda")
    assert _fwd_ex(d, p, ref_o, ref_l, ws, 0) == 0
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status(ws) == 0

    # the injected fault: the call itself launches fine, the device reports the timeout
    sentinel = torch.full_like(ref_o, 7.0)
    lse = torch.full_like(ref_l, 7.0)
    assert _fwd_ex(d, p, sentinel, lse, ws, NSA_TEST_SKIP_ARRIVE | NSA_TEST_SHORT_WAITS) == 0
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status(ws) == NSA_ERR_TIMEOUT
    assert bool((sentinel == 7.0).all()) and bool((lse == 7.0).all())   # outputs untouched

    # short waits alone change nothing on a healthy run
    o2 = torch.empty_like(ref_o)
    l2 = torch.empty_like(ref_l)
    assert _fwd_ex(d, p, o2, l2, ws, NSA_TEST_SHORT_WAITS) == 0
    torch.cuda.synchronize()
    assert nsa.nsa_sel_check_status(ws) == 0
    assert torch.equal(o2, ref_o) and torch.equal(l2, ref_l)

    # the next ordinary calls are exact
    for _ in range(3):
        o3, l3 = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], 64, p.scale,
                                      workspace=ws)
        torch.cuda.synchronize()
        assert nsa.nsa_sel_check_status(ws) == 0
        assert torch.equal(o3, ref_o) and torch.equal(l3, ref_l)

