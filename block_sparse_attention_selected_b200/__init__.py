"""NSA selected-block attention on B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/nsa_sel.h`` (``libnsa_sel.so``,
built in this directory by ``build.py``).  Functions carry the C names and only
marshal arguments: every step of the computation runs in the CUDA library.  There
is no fallback: if the library or a CUDA device is missing, calls raise.

Tensors: q [T, hq, 128], k/v [T, hkv, 128] bf16 CUDA; cu_seqlens int32 [nseq+1];
block_idx int32 [T, hkv, topk] (block numbers local to each sequence, -1 pads).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# NSA_SEL_LIBRARY=checks loads the bounds-checking build (libnsa_sel_checks.so) instead
LIB_PATH = os.path.join(_HERE, "libnsa_sel_checks.so" if os.environ.get("NSA_SEL_LIBRARY") == "checks"
                        else "libnsa_sel.so")

NSA_OK = 0
STATUS_NAMES = {0: "NSA_OK", 1: "NSA_ERR_INVALID_ARG", 2: "NSA_ERR_UNSUPPORTED",
                3: "NSA_ERR_WORKSPACE", 4: "NSA_ERR_CUDA", 5: "NSA_ERR_TIMEOUT",
                6: "NSA_ERR_BAD_INDEX", 7: "NSA_ERR_NO_DEVICE"}
EXPORTED = ["nsa_sel_attn_workspace_size", "nsa_sel_attn_fwd", "nsa_sel_attn_bwd",
            "nsa_sel_attn_fwd_profiled", "nsa_sel_attn_bwd_profiled", "nsa_sel_attn_fwd_ex",
            "nsa_sel_attn_bwd_ex", "nsa_sel_compress_kv", "nsa_sel_select_topk",
            "nsa_sel_block_scores", "nsa_sel_block_scores_workspace_size", "nsa_sel_bsfa_fwd",
            "nsa_sel_bsfa_workspace_size",
            "nsa_sel_invert_index",
            "nsa_sel_invert_index_noalloc", "nsa_sel_invert_index_noalloc_max_bytes",
            "nsa_sel_invert_index_scratch_bytes",
            "nsa_sel_validate_indices", "nsa_sel_check_status", "nsa_sel_status_string"]

_lib = None
_lock = threading.Lock()


class NsaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn}: {STATUS_NAMES.get(code, code)} ({_status_string(code)})")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads the CUDA library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(f"{path} is missing: build it with "
                                   "`python -m block_sparse_attention_selected_b200.build`")
            lib = ctypes.CDLL(path)
            P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            lib.nsa_sel_attn_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
            lib.nsa_sel_attn_workspace_size.restype = Z
            lib.nsa_sel_attn_fwd.argtypes = [P, P, P, P, I, I, I, I, I, P, I, I, F, P, P, P, Z, P]
            lib.nsa_sel_attn_fwd.restype = I
            lib.nsa_sel_attn_bwd.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P, I, I, F,
                                             P, P, P, P, Z, P]
            lib.nsa_sel_attn_bwd.restype = I
            IP = ctypes.POINTER(ctypes.c_int)
            lib.nsa_sel_attn_fwd_profiled.argtypes = lib.nsa_sel_attn_fwd.argtypes + [P, I, IP]
            lib.nsa_sel_attn_fwd_profiled.restype = I
            lib.nsa_sel_attn_bwd_profiled.argtypes = lib.nsa_sel_attn_bwd.argtypes + [P, I, IP]
            lib.nsa_sel_attn_bwd_profiled.restype = I
            lib.nsa_sel_attn_fwd_ex.argtypes = lib.nsa_sel_attn_fwd.argtypes + [ctypes.c_uint, I, P, I, IP]
            lib.nsa_sel_attn_fwd_ex.restype = I
            lib.nsa_sel_attn_bwd_ex.argtypes = lib.nsa_sel_attn_bwd.argtypes + [ctypes.c_uint, I, P, I, IP]
            lib.nsa_sel_attn_bwd_ex.restype = I
            lib.nsa_sel_compress_kv.argtypes = [P, P, P, I, I, I, I, I, I, ctypes.c_uint, P, P, P, P]
            lib.nsa_sel_compress_kv.restype = I
            lib.nsa_sel_select_topk.argtypes = [P, P, I, I, I, I, I, I, I, I, P, P, Z, P]
            lib.nsa_sel_select_topk.restype = I
            lib.nsa_sel_block_scores_workspace_size.argtypes = [I]
            lib.nsa_sel_block_scores_workspace_size.restype = Z
            lib.nsa_sel_block_scores.argtypes = [P, P, I, P, P, I, I, I, I, I, I, I, I, F, I, P, P, Z, P]
            lib.nsa_sel_block_scores.restype = I
            lib.nsa_sel_bsfa_workspace_size.argtypes = [I]
            lib.nsa_sel_bsfa_workspace_size.restype = Z
            lib.nsa_sel_bsfa_fwd.argtypes = [P, P, P, P, I, I, I, I, I, I, F, P, P, P, P, Z, P]
            lib.nsa_sel_bsfa_fwd.restype = I
            lib.nsa_sel_invert_index.argtypes = [P, I, I, I, P, I, I, P, P, P, P, Z, P]
            lib.nsa_sel_invert_index.restype = I
            lib.nsa_sel_invert_index_noalloc.argtypes = [P, I, I, I, P, I, I, P, P, P, P]
            lib.nsa_sel_invert_index_noalloc.restype = I
            lib.nsa_sel_invert_index_noalloc_max_bytes.argtypes = []
            lib.nsa_sel_invert_index_noalloc_max_bytes.restype = Z
            lib.nsa_sel_invert_index_scratch_bytes.argtypes = [I, I, I, I, I]
            lib.nsa_sel_invert_index_scratch_bytes.restype = Z
            lib.nsa_sel_validate_indices.argtypes = [P, I, I, I, P, I, I, P, P, P, Z, P]
            lib.nsa_sel_validate_indices.restype = I
            lib.nsa_sel_check_status.argtypes = [P, P]
            lib.nsa_sel_check_status.restype = I
            lib.nsa_sel_status_string.argtypes = [I]
            lib.nsa_sel_status_string.restype = ctypes.c_char_p
            _lib = lib
    return _lib


def _status_string(code: int) -> str:
    try:
        return load_library().nsa_sel_status_string(code).decode()
    except Exception:  # pragma: no cover
        return "?"


def _check(fn: str, code: int):
    if code != NSA_OK:
        raise NsaError(fn, code)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, name, dtype, ndim=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_ws_cache: dict = {}


def nsa_sel_attn_workspace_size(total_tokens, num_seqs, hq, hkv, head_dim, topk, block_size,
                                for_bwd=False) -> int:
    n = load_library().nsa_sel_attn_workspace_size(total_tokens, num_seqs, hq, hkv, head_dim,
                                                   topk, block_size, int(bool(for_bwd)))
    if n == 0:
        raise NsaError("nsa_sel_attn_workspace_size", 2)
    return int(n)


def _ws_key(dev: torch.device):
    # one cached workspace per (device, stream): calls on different streams may overlap
    # on the GPU and must not share scratch memory
    return (dev, torch.cuda.current_stream(dev).cuda_stream)


def get_workspace(nbytes: int, device) -> torch.Tensor:
    """A cached uint8 device buffer of at least nbytes (grown on demand) for the
    device's current stream; it is allocated on that stream, so the caching allocator
    orders its reuse after the calls that used it."""
    dev = torch.device(device)
    key = _ws_key(dev)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        _ws_cache.pop(key, None)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        _ws_cache[key] = ws
    return ws


def release_workspaces():
    _ws_cache.clear()


def _shapes(q, k, cu_seqlens, block_idx):
    T, hq, d = q.shape
    hkv = k.shape[1]
    topk = block_idx.shape[2]
    return T, hq, hkv, d, topk, cu_seqlens.numel() - 1


NSA_BWD_REUSE_INDEX = 1
NSA_F16 = 2


def _elem_type(q):
    """bf16 or fp16 attention tensors (the flag of the _ex calls)."""
    if q.dtype == torch.bfloat16:
        return torch.bfloat16, 0
    if q.dtype == torch.float16:
        return torch.float16, NSA_F16
    raise TypeError(f"q: expected bfloat16 or float16, got {q.dtype}")


def nsa_sel_attn_fwd(q, k, v, cu_seqlens, block_idx, block_size, scale=None, out=None, lse=None,
                     workspace=None, with_lse=True, window_size=0):
    """Forward selected attention; returns (out [T,hq,d], lse fp32 [hq,T]).

    q, k, v (and out) are all bf16 or all fp16.  with_lse=False: a forward with no
    backward to follow; the LSE is not stored and None is returned in its place.
    window_size > 0: keys must also lie in the last window_size positions up to the
    query's own (a sliding window on top of the selected blocks)."""
    dev = q.device
    et, flag = _elem_type(q)
    _need(q, "q", et, 3, dev)
    _need(k, "k", et, 3, dev)
    _need(v, "v", et, 3, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1, dev)
    _need(block_idx, "block_idx", torch.int32, 3, dev)
    T, hq, hkv, d, topk, nseq = _shapes(q, k, cu_seqlens, block_idx)
    if k.shape != (T, hkv, d) or v.shape != (T, hkv, d) or block_idx.shape[:2] != (T, hkv):
        raise ValueError("inconsistent shapes")
    scale = float(d ** -0.5 if scale is None else scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and with_lse:
        lse = torch.empty((hq, T), dtype=torch.float32, device=dev)
    _need(out, "out", et, 3, dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, 2, dev)
    nbytes = nsa_sel_attn_workspace_size(T, nseq, hq, hkv, d, topk, block_size, False)
    ws = workspace if workspace is not None else get_workspace(nbytes, dev)
    with torch.cuda.device(dev):
        _check("nsa_sel_attn_fwd", load_library().nsa_sel_attn_fwd_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), nseq, T, hq, hkv, d, _ptr(block_idx), topk,
            block_size, scale, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(dev), flag,
            int(window_size), None, 0, None))
    return out, lse


def nsa_sel_attn_bwd(q, k, v, out, lse, dout, cu_seqlens, block_idx, block_size, scale=None,
                     dq=None, dk=None, dv=None, workspace=None, reuse_index=False,
                     window_size=0):
    """Backward; returns (dq, dk, dv) in the type of q (bf16 or fp16).

    window_size: the forward's sliding window (0: none).

    reuse_index: `workspace` (sized for the backward) was given to the forward call for
    the same cu_seqlens / block_idx tensors and is reused untouched since; the backward
    then skips the index inversion (nsa_sel_attn_bwd_ex with NSA_BWD_REUSE_INDEX)."""
    dev = q.device
    et, flag = _elem_type(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, n, et, 3, dev)
    _need(lse, "lse", torch.float32, 2, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1, dev)
    _need(block_idx, "block_idx", torch.int32, 3, dev)
    T, hq, hkv, d, topk, nseq = _shapes(q, k, cu_seqlens, block_idx)
    scale = float(d ** -0.5 if scale is None else scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, n, et, 3, dev)
    nbytes = nsa_sel_attn_workspace_size(T, nseq, hq, hkv, d, topk, block_size, True)
    if reuse_index and workspace is None:
        raise ValueError("reuse_index needs the workspace the forward used")
    ws = workspace if workspace is not None else get_workspace(nbytes, dev)
    with torch.cuda.device(dev):
        _check("nsa_sel_attn_bwd", load_library().nsa_sel_attn_bwd_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(cu_seqlens), nseq, T,
            hq, hkv, d, _ptr(block_idx), topk, block_size, scale, _ptr(dq), _ptr(dk), _ptr(dv),
            _ptr(ws), ws.numel(), _stream(dev), (NSA_BWD_REUSE_INDEX if reuse_index else 0) | flag,
            int(window_size), None, 0, None))
    return dq, dk, dv


def nsa_sel_invert_index(cu_seqlens, block_idx, block_size, workspace=None):
    """The block-index inversion; returns (offsets int32 [hkv*NB+1], entries int32 [n])."""
    dev = block_idx.device
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1, dev)
    _need(block_idx, "block_idx", torch.int32, 3, dev)
    T, hkv, topk = block_idx.shape
    nseq = cu_seqlens.numel() - 1
    nbytes = nsa_sel_attn_workspace_size(T, nseq, hkv, hkv, 128, topk, block_size, False)
    ws = workspace if workspace is not None else get_workspace(nbytes, dev)
    offsets = torch.empty(hkv * (T // block_size + nseq) + 1, dtype=torch.int32, device=dev)
    entries = torch.empty(max(T * hkv * topk, 1), dtype=torch.int32, device=dev)
    counts = torch.zeros(2, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check("nsa_sel_invert_index", load_library().nsa_sel_invert_index(
            _ptr(cu_seqlens), nseq, T, hkv, _ptr(block_idx), topk, block_size, _ptr(offsets),
            _ptr(entries), _ptr(counts), _ptr(ws), ws.numel(), _stream(dev)))
    nb, n = (int(x) for x in counts.tolist())
    return offsets[:hkv * nb + 1], entries[:n]


def nsa_sel_invert_index_noalloc(cu_seqlens, block_idx, block_size):
    """The block-index inversion without a caller workspace.

    For callers that cannot allocate device memory (a plug-in inside a framework
    that owns all device memory, or a loop where cudaMalloc is not allowed): the
    library uses a fixed device array of its own as scratch.  Output buffers are
    still the caller's.  Calls sharing a device must not overlap on the GPU.
    Returns (offsets int32 [hkv*NB+1], entries int32 [n]).
    """
    dev = block_idx.device
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1, dev)
    _need(block_idx, "block_idx", torch.int32, 3, dev)
    T, hkv, topk = block_idx.shape
    nseq = cu_seqlens.numel() - 1
    offsets = torch.empty(hkv * (T // block_size + nseq) + 1, dtype=torch.int32, device=dev)
    entries = torch.empty(max(T * hkv * topk, 1), dtype=torch.int32, device=dev)
    counts = torch.zeros(2, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check("nsa_sel_invert_index_noalloc", load_library().nsa_sel_invert_index_noalloc(
            _ptr(cu_seqlens), nseq, T, hkv, _ptr(block_idx), topk, block_size, _ptr(offsets),
            _ptr(entries), _ptr(counts), _stream(dev)))
    nb, n = (int(x) for x in counts.tolist())
    return offsets[:hkv * nb + 1], entries[:n]


def nsa_sel_validate_indices(cu_seqlens, block_idx, block_size, workspace=None):
    """(n_out_of_range, n_duplicates); synchronous."""
    dev = block_idx.device
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1, dev)
    _need(block_idx, "block_idx", torch.int32, 3, dev)
    T, hkv, topk = block_idx.shape
    ws = workspace if workspace is not None else get_workspace(256, dev)
    a, b = ctypes.c_longlong(0), ctypes.c_longlong(0)
    with torch.cuda.device(dev):
        code = load_library().nsa_sel_validate_indices(
            _ptr(cu_seqlens), cu_seqlens.numel() - 1, T, hkv, _ptr(block_idx), topk, block_size,
            ctypes.byref(a), ctypes.byref(b), _ptr(ws), ws.numel(), _stream(dev))
    if code not in (0, 6):
        raise NsaError("nsa_sel_validate_indices", code)
    return int(a.value), int(b.value)


def nsa_sel_compress_kv(k, v, cu_seqlens, kernel_size=32, kernel_stride=16):
    """Mean-pooled compressed K and V of the selection step; returns (k_cmp, v_cmp,
    cu_cmp): k_cmp / v_cmp [floor(T / stride), hkv, d] in the type of k (rows past
    cu_cmp[-1] unused), cu_cmp int32 [nseq + 1]."""
    dev = k.device
    et, flag = _elem_type(k)
    _need(k, "k", et, 3, dev)
    _need(v, "v", et, 3, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1, dev)
    T, hkv, d = k.shape
    if v.shape != k.shape:
        raise ValueError("inconsistent shapes")
    nseq = cu_seqlens.numel() - 1
    rows = max(T // kernel_stride, 1)
    kc = torch.empty((rows, hkv, d), dtype=et, device=dev)
    vc = torch.empty((rows, hkv, d), dtype=et, device=dev)
    cu_cmp = torch.empty(nseq + 1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check("nsa_sel_compress_kv", load_library().nsa_sel_compress_kv(
            _ptr(k), _ptr(v), _ptr(cu_seqlens), nseq, T, hkv, d, kernel_size, kernel_stride, flag,
            _ptr(kc), _ptr(vc), _ptr(cu_cmp), _stream(dev)))
    return kc, vc, cu_cmp


def nsa_sel_block_scores(q, k_cmp, cu_seqlens, cu_cmp, block_size, nb_stride, scale=None,
                         kernel_size=32, kernel_stride=16, workspace=None):
    """Selection-block scores fp32 [T, hkv, nb_stride] from attention over the compressed
    keys (entries past each row's own block are left uninitialised)."""
    dev = q.device
    _need(q, "q", torch.bfloat16, 3, dev)
    _need(k_cmp, "k_cmp", torch.bfloat16, 3, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1, dev)
    _need(cu_cmp, "cu_cmp", torch.int32, 1, dev)
    T, hq, d = q.shape
    rows, hkv, _ = k_cmp.shape
    scale = float(d ** -0.5 if scale is None else scale)
    nseq = cu_seqlens.numel() - 1
    lib = load_library()
    nbytes = int(lib.nsa_sel_block_scores_workspace_size(nseq))
    ws = workspace if workspace is not None else get_workspace(nbytes, dev)
    scores = torch.empty((T, hkv, nb_stride), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check("nsa_sel_block_scores", lib.nsa_sel_block_scores(
            _ptr(q), _ptr(k_cmp), rows, _ptr(cu_seqlens), _ptr(cu_cmp), nseq, T, hq, hkv, d,
            block_size, kernel_size, kernel_stride, scale, nb_stride, _ptr(scores), _ptr(ws),
            ws.numel(), _stream(dev)))
    return scores


def nsa_sel_select_blocks(q, k, v, cu_seqlens, block_size=64, topk=16, init_blocks=1,
                          local_blocks=2, max_seqlen=None, scale=None):
    """The whole selection step on the GPU: compression, block scores, top-k; returns
    block_idx int32 [T, hkv, topk].  max_seqlen (host int) sizes the score rows."""
    T = q.shape[0]
    L = int(max_seqlen) if max_seqlen is not None else T
    nb_stride = max((L + block_size - 1) // block_size, 1)
    kc, _, cu_cmp = nsa_sel_compress_kv(k, v, cu_seqlens)
    sc = nsa_sel_block_scores(q, kc, cu_seqlens, cu_cmp, block_size, nb_stride, scale)
    return nsa_sel_select_topk(sc, cu_seqlens, block_size, topk, init_blocks, local_blocks)


def nsa_sel_bsfa_fwd(q, k, v, cu_seqlens, tau, scale=None, block_size=64, workspace=None):
    """Threshold-pruned block attention; returns (out bf16 [T, hq, d], lse fp32 [hq, T]).
    tau: fp32 [hq] thresholds on the device."""
    dev = q.device
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, 3, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1, dev)
    _need(tau, "tau", torch.float32, 1, dev)
    T, hq, d = q.shape
    hkv = k.shape[1]
    if tau.numel() != hq:
        raise ValueError("tau needs one threshold per query head")
    scale = float(d ** -0.5 if scale is None else scale)
    nseq = cu_seqlens.numel() - 1
    lib = load_library()
    ws = workspace if workspace is not None else get_workspace(int(lib.nsa_sel_bsfa_workspace_size(nseq)), dev)
    out = torch.empty_like(q)
    lse = torch.empty((hq, T), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check("nsa_sel_bsfa_fwd", lib.nsa_sel_bsfa_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), nseq, T, hq, hkv, d, block_size, scale,
            _ptr(tau), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(dev)))
    return out, lse


def nsa_sel_select_topk(scores, cu_seqlens, block_size, topk, init_blocks=1, local_blocks=2,
                        workspace=None):
    """block_idx int32 [T, hkv, topk] from block scores fp32 [T, hkv, nb_stride]."""
    dev = scores.device
    _need(scores, "scores", torch.float32, 3, dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1, dev)
    T, hkv, nb = scores.shape
    out = torch.empty((T, hkv, topk), dtype=torch.int32, device=dev)
    ws = workspace if workspace is not None else get_workspace(256, dev)
    with torch.cuda.device(dev):
        _check("nsa_sel_select_topk", load_library().nsa_sel_select_topk(
            _ptr(scores), _ptr(cu_seqlens), cu_seqlens.numel() - 1, T, hkv, nb, block_size, topk,
            init_blocks, local_blocks, _ptr(out), _ptr(ws), ws.numel(), _stream(dev)))
    return out


def nsa_sel_check_status(workspace=None, device=None) -> int:
    """Device-side status of the last call that used this workspace (synchronises); by
    default the cached workspace of the device's current stream."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    ws = workspace if workspace is not None else _ws_cache.get(_ws_key(dev))
    if ws is None:
        return NSA_OK
    with torch.cuda.device(ws.device):
        return int(load_library().nsa_sel_check_status(_ptr(ws), _stream(ws.device)))


class SelectedAttention(torch.autograd.Function):
    """Autograd wrapper: forward saves LSE, backward returns dQ, dK, dV."""

    @staticmethod
    def forward(ctx, q, k, v, cu_seqlens, block_idx, block_size, scale, window_size=0):
        out, lse = nsa_sel_attn_fwd(q, k, v, cu_seqlens, block_idx, block_size, scale,
                                    window_size=window_size)
        ctx.save_for_backward(q, k, v, out, lse, cu_seqlens, block_idx)
        ctx.block_size, ctx.scale, ctx.window_size = block_size, scale, window_size
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse, cu, bi = ctx.saved_tensors
        dq, dk, dv = nsa_sel_attn_bwd(q, k, v, out, lse, dout.contiguous(), cu, bi,
                                      ctx.block_size, ctx.scale, window_size=ctx.window_size)
        return dq, dk, dv, None, None, None, None, None


def selected_attention(q, k, v, cu_seqlens, block_idx, block_size=64, scale=None, window_size=0):
    return SelectedAttention.apply(q, k, v, cu_seqlens, block_idx, block_size,
                                   float(q.shape[-1] ** -0.5 if scale is None else scale),
                                   int(window_size))
