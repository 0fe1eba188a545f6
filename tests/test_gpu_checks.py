"""The bounds-checking build (libnsa_sel_checks.so, compiled with -DNSA_SEL_CHECKS).

It checks every gathered row and K/V block coordinate before issuing the copy and
records NSA_ERR_BAD_INDEX instead of reading out of bounds.  On valid inputs it must
raise no error and give the ordinary build's results bit for bit; it runs in a child
process, since a process loads one of the two libraries.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import block_sparse_attention_selected_b200 as nsa
import nsa_inputs as ni
from block_sparse_attention_selected_b200 import build as nsa_build
from gpu_util import to_device

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import block_sparse_attention_selected_b200 as nsa, nsa_inputs as ni
from gpu_util import to_device
assert nsa.LIB_PATH.endswith("libnsa_sel_checks.so")
p = ni.make_problem([1500, 300, 1], hq=8, hkv=2, block_size=64, topk=16, seed=97)
d = to_device(p)
out, lse = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], 64, p.scale)
dq, dk, dv = nsa.nsa_sel_attn_bwd(d["q"], d["k"], d["v"], out, lse, d["dout"], d["cu"], d["bidx"], 64, p.scale)
torch.cuda.synchronize()
st = nsa.nsa_sel_check_status()
np.savez(sys.argv[2], st=st, **{k: v.float().cpu().numpy() for k, v in
         dict(out=out, lse=lse, dq=dq, dk=dk, dv=dv).items()})
"""


def test_checking_build_matches_and_reports_nothing(tmp_path):
    nsa_build.build(checks=True)
    path = str(tmp_path / "checks.npz")
    env = dict(os.environ, NSA_SEL_LIBRARY="checks")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, path], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    got = np.load(path)
    assert int(got["st"]) == 0
    p = ni.make_problem([1500, 300, 1], hq=8, hkv=2, block_size=64, topk=16, seed=97)
    d = to_device(p)
    out, lse = nsa.nsa_sel_attn_fwd(d["q"], d["k"], d["v"], d["cu"], d["bidx"], 64, p.scale)
    dq, dk, dv = nsa.nsa_sel_attn_bwd(d["q"], d["k"], d["v"], out, lse, d["dout"], d["cu"],
                                      d["bidx"], 64, p.scale)
    torch.cuda.synchronize()
    for name, t in dict(out=out, lse=lse, dq=dq, dk=dk, dv=dv).items():
        assert np.array_equal(got[name], t.float().cpu().numpy()), name
