"""The C ABI library builds, loads and exports every symbol of include/nsa_sel.h.

CPU only: no call here reaches a CUDA kernel.  Argument checks run on the host
before any device work, so their error codes can be checked without a GPU.
"""
import ctypes
import os
import re

import pytest

import block_sparse_attention_selected_b200 as nsa
from block_sparse_attention_selected_b200 import build as nsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nsa_sel.h")


@pytest.fixture(scope="module")
def lib():
    nsa_build.build()
    return nsa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nsa_sel_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(nsa.EXPORTED)


def test_status_strings(lib):
    for code in range(8):
        s = lib.nsa_sel_status_string(code)
        assert s and s != b"unknown status"
    assert lib.nsa_sel_status_string(99) == b"unknown status"


def test_workspace_size_domain(lib):
    ws = nsa.nsa_sel_attn_workspace_size
    base = ws(65536, 1, 16, 4, 128, 16, 64, False)
    # partial results dominate: T * hq * topk rows of 128 bf16 + one fp32
    assert base >= 65536 * 16 * 16 * (256 + 4)
    assert ws(65536, 1, 16, 4, 128, 16, 64, True) > base
    assert ws(0, 1, 4, 4, 128, 8, 64, False) > 0
    f = lib.nsa_sel_attn_workspace_size
    assert f(1024, 1, 4, 4, 64, 8, 64, 0) > 0           # head_dim 64: forward
    # ... and the backward, whose dQ partials keep 128 columns
    assert f(1024, 1, 4, 4, 64, 8, 64, 1) >= f(1024, 1, 4, 4, 128, 8, 64, 1)
    assert f(1024, 1, 4, 4, 256, 8, 64, 0) > 0          # head_dim 256 with block 64: forward
    assert f(1024, 1, 4, 4, 256, 8, 128, 0) == 0        # ... not with block 128
    assert f(1024, 1, 4, 4, 256, 8, 64, 1) == 0         # ... and no backward
    assert f(1024, 1, 4, 4, 96, 8, 64, 0) == 0          # head_dim 96 not supported
    assert f(1024, 1, 4, 4, 64, 8, 64, 0) < f(1024, 1, 4, 4, 256, 8, 64, 0)   # partial rows of 2 d bytes
    assert f(1024, 1, 4, 4, 128, 8, 32, 0) == 0         # block 32 not supported
    assert f(1024, 1, 4, 4, 128, 65, 64, 0) == 0        # topk > 64
    assert f(1024, 1, 64, 2, 128, 8, 64, 0) > 0         # group 32 fills a tile with 4 tokens
    assert f(1024, 1, 256, 1, 128, 8, 64, 0) == 0       # group 256 > 128 rows of a tile
    assert f(1024, 1, 6, 2, 128, 8, 64, 0) == 0         # group 3 does not divide 128
    assert f(1024, 1, 6, 4, 128, 8, 64, 0) == 0         # hq % hkv != 0
    assert f(1 << 25, 1, 4, 4, 128, 8, 64, 0) == 0      # too many tokens
    # 2^22 tokens of 128 heads over one KV head, top-64: 2^35 forward partial rows,
    # beyond 32-bit row coordinates (and any device memory)
    assert f(1 << 22, 1, 128, 1, 128, 64, 64, 0) == 0
    assert f(1 << 16, 1, 128, 1, 128, 64, 64, 0) > 0


def test_host_argument_errors(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)           # never dereferenced: checks fail first
    # unsupported head_dim (96; and 256 with block 128)
    rc = lib.nsa_sel_attn_fwd(fake, fake, fake, fake, 1, 64, 4, 4, 96, fake, 8, 64, 0.1,
                              fake, fake, fake, 1 << 30, None)
    assert rc == 2
    rc = lib.nsa_sel_attn_fwd(fake, fake, fake, fake, 1, 64, 4, 4, 256, fake, 8, 128, 0.1,
                              fake, fake, fake, 1 << 30, None)
    assert rc == 2
    # head_dim 256 in the backward
    rc = lib.nsa_sel_attn_bwd(fake, fake, fake, fake, fake, fake, fake, 1, 64, 4, 4, 256, fake, 8,
                              64, 0.1, fake, fake, fake, fake, 1 << 30, None)
    assert rc == 2
    # null cu_seqlens
    rc = lib.nsa_sel_attn_fwd(fake, fake, fake, None, 1, 64, 4, 4, 128, fake, 8, 64, 0.1,
                              fake, fake, fake, 1 << 30, None)
    assert rc == 1
    # workspace too small
    rc = lib.nsa_sel_attn_fwd(fake, fake, fake, fake, 1, 64, 4, 4, 128, fake, 8, 64, 0.1,
                              fake, fake, fake, 256, None)
    assert rc == 3
    # misaligned q
    rc = lib.nsa_sel_attn_fwd(P((1 << 20) + 2), fake, fake, fake, 1, 64, 4, 4, 128, fake, 8, 64,
                              0.1, fake, fake, fake, 1 << 30, None)
    assert rc == 1
    # bad scale
    rc = lib.nsa_sel_attn_fwd(fake, fake, fake, fake, 1, 64, 4, 4, 128, fake, 8, 64, -1.0,
                              fake, fake, fake, 1 << 30, None)
    assert rc == 1
    # backward: hq % hkv
    rc = lib.nsa_sel_attn_bwd(fake, fake, fake, fake, fake, fake, fake, 1, 64, 6, 4, 128, fake,
                              8, 64, 0.1, fake, fake, fake, fake, 1 << 30, None)
    assert rc == 1
    # inversion: bad block size
    rc = lib.nsa_sel_invert_index(fake, 1, 64, 4, fake, 8, 96, fake, fake, fake, fake, 1 << 30,
                                  None)
    assert rc == 2
    assert lib.nsa_sel_check_status(None, None) == 1


def test_option_flags_checked_on_the_host(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)           # never dereferenced: the flag check comes first
    # forward: only NSA_F16 (2) is an option
    rc = lib.nsa_sel_attn_fwd_ex(fake, fake, fake, fake, 1, 64, 4, 4, 128, fake, 8, 64, 0.1,
                                 fake, fake, fake, 1 << 30, None, 1, 0, None, 0, None)
    assert rc == 1
    rc = lib.nsa_sel_attn_fwd_ex(fake, fake, fake, fake, 1, 64, 4, 4, 128, fake, 8, 64, 0.1,
                                 fake, fake, fake, 1 << 30, None, 4, 0, None, 0, None)
    assert rc == 1
    # backward: NSA_BWD_REUSE_INDEX (1) and NSA_F16 (2)
    rc = lib.nsa_sel_attn_bwd_ex(fake, fake, fake, fake, fake, fake, fake, 1, 64, 4, 4, 128,
                                 fake, 8, 64, 0.1, fake, fake, fake, fake, 1 << 30, None, 8,
                                 0, None, 0, None)
    assert rc == 1
    # a valid flag still reaches the usual argument checks (here: head_dim 256)
    rc = lib.nsa_sel_attn_bwd_ex(fake, fake, fake, fake, fake, fake, fake, 1, 64, 4, 4, 256,
                                 fake, 8, 64, 0.1, fake, fake, fake, fake, 1 << 30, None, 3,
                                 0, None, 0, None)
    assert rc == 2
    # a negative sliding window is an argument error in both directions
    rc = lib.nsa_sel_attn_fwd_ex(fake, fake, fake, fake, 1, 64, 4, 4, 128, fake, 8, 64, 0.1,
                                 fake, fake, fake, 1 << 30, None, 0, -1, None, 0, None)
    assert rc == 1
    rc = lib.nsa_sel_attn_bwd_ex(fake, fake, fake, fake, fake, fake, fake, 1, 64, 4, 4, 128,
                                 fake, 8, 64, 0.1, fake, fake, fake, fake, 1 << 30, None, 0,
                                 -5, None, 0, None)
    assert rc == 1
    assert nsa.NSA_BWD_REUSE_INDEX == 1 and nsa.NSA_F16 == 2


def test_selection_entry_points_check_arguments(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)           # never dereferenced: the checks come first
    # compress: a kernel shorter than its stride, a head dim other than 128, a bad flag
    assert lib.nsa_sel_compress_kv(fake, fake, fake, 1, 64, 2, 128, 8, 16, 0, fake, fake, fake,
                                   None) == 1
    assert lib.nsa_sel_compress_kv(fake, fake, fake, 1, 64, 2, 64, 32, 16, 0, fake, fake, fake,
                                   None) == 2
    assert lib.nsa_sel_compress_kv(fake, fake, fake, 1, 64, 2, 128, 32, 16, 4, fake, fake, fake,
                                   None) == 1
    # top-k: topk 0, more than 64 slots, score rows over 1024 blocks, a short workspace
    assert lib.nsa_sel_select_topk(fake, fake, 1, 64, 2, 8, 64, 0, 1, 2, fake, fake, 1 << 20,
                                   None) == 1
    assert lib.nsa_sel_select_topk(fake, fake, 1, 64, 2, 8, 64, 65, 1, 2, fake, fake, 1 << 20,
                                   None) == 2
    assert lib.nsa_sel_select_topk(fake, fake, 1, 64, 2, 1025, 64, 16, 1, 2, fake, fake, 1 << 20,
                                   None) == 2
    assert lib.nsa_sel_select_topk(fake, fake, 1, 64, 2, 8, 64, 16, 1, 2, fake, fake, 128,
                                   None) == 3


def test_block_scores_entry_point_checks_arguments(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)
    F = ctypes.c_float
    ws = lib.nsa_sel_block_scores_workspace_size(3)
    assert ws >= 256 + 16 and lib.nsa_sel_block_scores_workspace_size(0) == 0
    args = lambda hq, hkv, bs, ksz, kst, rows, wsb: (fake, fake, rows, fake, fake, 3, 256, hq, hkv,
                                                     128, bs, ksz, kst, F(0.1), 8, fake, fake, wsb,
                                                     None)
    assert lib.nsa_sel_block_scores(*args(12, 4, 64, 32, 16, 16, ws)) == 2   # group 3
    assert lib.nsa_sel_block_scores(*args(128, 2, 64, 32, 16, 16, ws)) == 2  # group 64 > 32
    assert lib.nsa_sel_block_scores(*args(8, 2, 64, 16, 16, 16, ws)) == 2    # other geometry
    assert lib.nsa_sel_block_scores(*args(8, 2, 32, 32, 16, 16, ws)) == 2    # block 32
    assert lib.nsa_sel_block_scores(*args(8, 2, 64, 32, 16, 0, ws)) == 1     # no compressed rows
    assert lib.nsa_sel_block_scores(*args(8, 2, 64, 32, 16, 16, 100)) == 3   # short workspace


def test_bsfa_entry_point_checks_arguments(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)
    F = ctypes.c_float
    ws = lib.nsa_sel_bsfa_workspace_size(2)
    a = lambda hq, hkv, d, bs, wsb: (fake, fake, fake, fake, 2, 256, hq, hkv, d, bs, F(0.1), fake,
                                     fake, fake, fake, wsb, None)
    assert lib.nsa_sel_bsfa_fwd(*a(12, 4, 128, 64, ws)) == 2      # group 3
    assert lib.nsa_sel_bsfa_fwd(*a(8, 2, 64, 64, ws)) == 2        # head dim 64
    assert lib.nsa_sel_bsfa_fwd(*a(8, 2, 128, 128, ws)) == 2      # block 128
    assert lib.nsa_sel_bsfa_fwd(*a(8, 3, 128, 64, ws)) == 1       # hq % hkv
    assert lib.nsa_sel_bsfa_fwd(*a(8, 2, 128, 64, 64)) == 3       # short workspace


def test_binding_rejects_other_element_types():
    import torch
    x = torch.zeros((4, 2, 128), dtype=torch.float32)
    with pytest.raises(TypeError):
        nsa._elem_type(x)
    assert nsa._elem_type(x.to(torch.float16))[1] == nsa.NSA_F16
    assert nsa._elem_type(x.to(torch.bfloat16))[1] == 0


def test_product_path_has_no_oracle_dependency():
    """The package and its sources never import, link or call the oracle."""
    pkg = os.path.join(ROOT, "block_sparse_attention_selected_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in src.lower().replace("oracle_", ""), f


def test_cached_workspace_is_per_stream(monkeypatch):
    """Host logic of the binding's workspace cache, with the CUDA calls faked: one buffer
    per (device, stream), grown on demand, reused on the same stream."""
    import types
    import torch
    current = {"s": 11}
    monkeypatch.setattr(torch.cuda, "current_stream",
                        lambda dev=None: types.SimpleNamespace(cuda_stream=current["s"]))
    real_empty = torch.empty
    monkeypatch.setattr(torch, "empty", lambda n, dtype=None, device=None: real_empty(n, dtype=dtype))
    nsa.release_workspaces()
    dev = torch.device("cuda", 0)
    a = nsa.get_workspace(100, dev)
    assert nsa.get_workspace(50, dev) is a                  # same stream: reused
    current["s"] = 22
    b = nsa.get_workspace(50, dev)
    assert b is not a                                       # another stream: its own buffer
    current["s"] = 11
    c = nsa.get_workspace(400, dev)
    assert c is not a and c.numel() >= 400                  # grown on demand
    assert nsa.get_workspace(10, dev) is c
    current["s"] = 22
    assert nsa.get_workspace(10, dev) is b
    nsa.release_workspaces()


def test_binding_makes_the_tensors_device_current():
    """Every call into the library runs with the tensors' device current: the C side
    launches on, and takes the no-allocation scratch of, the current device, and
    rejects a stream of another device."""
    import ast
    import inspect
    tree = ast.parse(inspect.getsource(nsa))
    calls = 0

    def guarded(node, parents):
        for p in parents:
            if isinstance(p, ast.With) and any(
                    isinstance(it.context_expr, ast.Call) and
                    ast.unparse(it.context_expr.func) == "torch.cuda.device" for it in p.items):
                return True
        return False

    def visit(node, parents):
        nonlocal calls
        if isinstance(node, ast.Call) and isinstance(node.func, ast.Attribute) and \
                node.func.attr.startswith("nsa_sel_") and \
                not node.func.attr.endswith(("_size", "_max_bytes", "_string")):
            base = ast.unparse(node.func.value)
            if base in ("lib", "load_library()"):
                calls += 1
                assert guarded(node, parents), f"{node.func.attr} at line {node.lineno}"
        for ch in ast.iter_child_nodes(node):
            visit(ch, parents + [node])

    visit(tree, [])
    assert calls >= 10


def test_test_only_flags_are_forward_only(lib):
    """The fault-injection options exist for the forward's failure-detection test only;
    the backward rejects them on the host, before any device work."""
    rc = lib.nsa_sel_attn_bwd_ex(*([None] * 7), 1, 0, 1, 1, 128, None, 1, 64, ctypes.c_float(0.1),
                                 None, None, None, None, 0, None, 0x200, 0, None, 0, None)
    assert rc == 1   # NSA_ERR_INVALID_ARG
    rc = lib.nsa_sel_attn_fwd_ex(*([None] * 4), 1, 0, 1, 1, 128, None, 1, 64, ctypes.c_float(0.1),
                                 None, None, None, 0, None, 0x400, 0, None, 0, None)
    assert rc == 1   # an unknown bit


def test_noalloc_size_boundary(lib):
    """The no-allocation inversion takes exactly the sizes whose scratch (as reported by
    nsa_sel_invert_index_scratch_bytes) fits its fixed array: the largest such size
    passes the size check (and then, without a GPU, stops at the device check), the
    next one is refused with NSA_ERR_WORKSPACE before any device work."""
    limit = lib.nsa_sel_invert_index_noalloc_max_bytes()
    need = lib.nsa_sel_invert_index_scratch_bytes
    assert need(1000, 1, 4, 16, 64) > 1000 * 4 * 16 * 16
    assert need(1000, 1, 4, 16, 32) == 0                 # block 32: outside the domain
    lo, hi = 1, 1 << 22
    while lo < hi:                                       # largest T that fits
        mid = (lo + hi + 1) // 2
        if need(mid, 1, 4, 16, 64) <= limit:
            lo = mid
        else:
            hi = mid - 1
    P = ctypes.c_void_p
    fake = P(1 << 20)          # never dereferenced
    call = lambda T: lib.nsa_sel_invert_index_noalloc(fake, 1, T, 4, fake, 16, 64, fake, fake,
                                                      fake, None)
    assert call(lo + 1) == 3                             # NSA_ERR_WORKSPACE
    assert call(lo) != 3                                 # past the size check
