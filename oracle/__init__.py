"""fp64 CPU oracle for NSA selected-block attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product path (the CUDA
library and its binding) never does, and shares no code with it.

The arithmetic lives in ``nsa_oracle.c`` (plain C loops in double precision);
this module compiles it with gcc on first use and marshals numpy arrays.

Parity status of each function (what pins it, see ``tests/test_oracle.py``):

* ``fwd``            pinned: dense-causal equivalence (vs torch float64 SDPA and a
                     dense loop), index-order invariance, weights sum to one,
                     brute force with an explicit mask, closed forms.
* ``bwd``            pinned: central finite differences, torch float64 autograd in
                     the dense-causal case, the identity D = <dO, O>.
* ``bwd_dq`` / ``bwd_dkdv_keys``  pinned against ``bwd`` (itself pinned).
* ``window`` (all four)  pinned: dense selection with a window against torch float64
                     SDPA / autograd under an explicit band mask, W = 1 closed form,
                     a window wider than every sequence changes nothing.
* ``invert``         pinned: brute-force nested loops on tiny inputs, round trip,
                     sortedness, counts.

The block-selection step that produces ``block_idx`` (compression, compressed
attention, block scores, top-k) is the numpy module ``oracle.selection``, pinned in
``tests/test_selection_oracle.py``; threshold-pruned block attention (BSFA) is
``oracle.bsfa``, pinned in ``tests/test_bsfa_oracle.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nsa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "libnsa_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2 -fopenmp); returns the .so path."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            L = ctypes.c_int64
            D = ctypes.c_double
            common = [P, P, P, P, I, I, I, I, P, I, I, D]
            lib.nsa_oracle_fwd.argtypes = common[:] + [P, L, P, P, L, I]
            lib.nsa_oracle_fwd.restype = I
            lib.nsa_oracle_bwd.argtypes = [P, P, P, P, P, I, I, I, I, P, I, I, D, P, P, P, L, I]
            lib.nsa_oracle_bwd.restype = I
            lib.nsa_oracle_bwd_dq.argtypes = [P, P, P, P, P, I, I, I, I, P, I, I, D, P, L, P, L, I]
            lib.nsa_oracle_bwd_dq.restype = I
            lib.nsa_oracle_bwd_dkdv_keys.argtypes = [P, P, P, P, P, I, I, I, I, P, I, I, D,
                                                     I, L, I, P, P, L, I]
            lib.nsa_oracle_bwd_dkdv_keys.restype = I
            lib.nsa_oracle_num_blocks.argtypes = [P, I, I]
            lib.nsa_oracle_num_blocks.restype = L
            lib.nsa_oracle_invert.argtypes = [P, I, I, P, I, I, P, P, L]
            lib.nsa_oracle_invert.restype = L
            _lib = lib
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _shape_args(q, k, cu, block_idx):
    T, hq, d = q.shape
    hkv = k.shape[1]
    topk = block_idx.shape[2]
    return T, hq, hkv, d, topk, len(cu) - 1


def fwd(q, k, v, cu_seqlens, block_idx, block_size, scale, tokens=None, nthreads=0, window=0):
    """O [ntok, hq, d] float64 and LSE [ntok, hq] float64 for the listed tokens.

    window > 0 restricts every query at local position i to keys j > i - window as well
    (a sliding window of that many positions, the query's own included)."""
    lib = _load()
    q, k, v = _f32(q), _f32(k), _f32(v)
    cu, bi = _i32(cu_seqlens), _i32(block_idx)
    T, hq, hkv, d, topk, nseq = _shape_args(q, k, cu, bi)
    toks = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    ntok = T if toks is None else len(toks)
    out = np.empty((ntok, hq, d), dtype=np.float64)
    lse = np.empty((ntok, hq), dtype=np.float64)
    rc = lib.nsa_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu), nseq, hq, hkv, d, _ptr(bi),
                            topk, block_size, float(scale), _ptr(toks), ntok, _ptr(out),
                            _ptr(lse), int(window), int(nthreads))
    if rc:
        raise RuntimeError(f"oracle fwd failed: {rc}")
    return out, lse


def bwd(q, k, v, dout, cu_seqlens, block_idx, block_size, scale, nthreads=0, window=0):
    """Full backward: dQ [T, hq, d], dK, dV [T, hkv, d] float64 (window as in fwd)."""
    lib = _load()
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(dout)
    cu, bi = _i32(cu_seqlens), _i32(block_idx)
    T, hq, hkv, d, topk, nseq = _shape_args(q, k, cu, bi)
    dq = np.empty((T, hq, d), dtype=np.float64)
    dk = np.empty((T, hkv, d), dtype=np.float64)
    dv = np.empty((T, hkv, d), dtype=np.float64)
    rc = lib.nsa_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(cu), nseq, hq, hkv, d,
                            _ptr(bi), topk, block_size, float(scale), _ptr(dq), _ptr(dk),
                            _ptr(dv), int(window), int(nthreads))
    if rc:
        raise RuntimeError(f"oracle bwd failed: {rc}")
    return dq, dk, dv


def bwd_dq(q, k, v, dout, cu_seqlens, block_idx, block_size, scale, tokens, nthreads=0,
           window=0):
    """dQ [ntok, hq, d] float64 for the listed tokens (window as in fwd)."""
    lib = _load()
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(dout)
    cu, bi = _i32(cu_seqlens), _i32(block_idx)
    T, hq, hkv, d, topk, nseq = _shape_args(q, k, cu, bi)
    toks = np.ascontiguousarray(tokens, dtype=np.int64)
    dq = np.empty((len(toks), hq, d), dtype=np.float64)
    rc = lib.nsa_oracle_bwd_dq(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(cu), nseq, hq, hkv, d,
                               _ptr(bi), topk, block_size, float(scale), _ptr(toks), len(toks),
                               _ptr(dq), int(window), int(nthreads))
    if rc:
        raise RuntimeError(f"oracle bwd_dq failed: {rc}")
    return dq


def bwd_dkdv_keys(q, k, v, dout, cu_seqlens, block_idx, block_size, scale, g, key0, nkeys,
                  nthreads=0, window=0):
    """dK, dV [nkeys, d] float64 of KV head g for keys key0 .. key0+nkeys-1 (one sequence;
    window as in fwd)."""
    lib = _load()
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(dout)
    cu, bi = _i32(cu_seqlens), _i32(block_idx)
    T, hq, hkv, d, topk, nseq = _shape_args(q, k, cu, bi)
    dk = np.empty((nkeys, d), dtype=np.float64)
    dv = np.empty((nkeys, d), dtype=np.float64)
    rc = lib.nsa_oracle_bwd_dkdv_keys(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(cu), nseq, hq,
                                      hkv, d, _ptr(bi), topk, block_size, float(scale), int(g),
                                      int(key0), int(nkeys), _ptr(dk), _ptr(dv), int(window),
                                      int(nthreads))
    if rc:
        raise RuntimeError(f"oracle bwd_dkdv_keys failed: {rc}")
    return dk, dv


def num_blocks(cu_seqlens, block_size) -> int:
    cu = _i32(cu_seqlens)
    return int(_load().nsa_oracle_num_blocks(_ptr(cu), len(cu) - 1, block_size))


def invert(cu_seqlens, block_idx, block_size):
    """(offsets int32 [hkv*NBtot+1], entries int32 [n]) with entry = t*64 + slot."""
    lib = _load()
    cu, bi = _i32(cu_seqlens), _i32(block_idx)
    T, hkv, topk = bi.shape
    nbk = hkv * num_blocks(cu, block_size)
    offsets = np.empty(nbk + 1, dtype=np.int32)
    n = lib.nsa_oracle_invert(_ptr(cu), len(cu) - 1, hkv, _ptr(bi), topk, block_size,
                              _ptr(offsets), None, 0)
    if n < 0:
        raise RuntimeError(f"oracle invert failed: {n}")
    entries = np.empty(max(int(n), 1), dtype=np.int32)
    n2 = lib.nsa_oracle_invert(_ptr(cu), len(cu) - 1, hkv, _ptr(bi), topk, block_size,
                               _ptr(offsets), _ptr(entries), len(entries))
    if n2 != n:
        raise RuntimeError(f"oracle invert failed: {n2}")
    return offsets, entries[:n]
