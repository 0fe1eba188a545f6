"""Helpers shared by the GPU parity tests (inputs to the device, sampling, metrics)."""
from __future__ import annotations

import numpy as np
import torch

import nsa_inputs as ni

# Tolerances for the bf16 path against the fp64 oracle.
TOL_O = 1e-2        # max |O_gpu - O_ref| beyond the bf16 quantisation of O_ref itself
TOL_LSE = 1e-3      # max |LSE_gpu - LSE_ref|
TOL_GRAD = 2e-2     # ||g_gpu - g_ref||_F / ||g_ref||_F for dQ, dK, dV


def to_device(p: ni.Problem, dev="cuda", dtype=torch.bfloat16):
    f = lambda a: torch.from_numpy(a).to(dev).to(dtype).contiguous()
    d = dict(q=f(p.q), k=f(p.k), v=f(p.v),
             cu=torch.from_numpy(p.cu_seqlens).to(dev),
             bidx=torch.from_numpy(np.ascontiguousarray(p.block_idx)).to(dev))
    if p.dout is not None:
        d["dout"] = f(p.dout)
    return d


def sample_tokens(cu_seqlens, block_size, n_random=96, seed=0):
    """Stratified token sample: sequence starts/ends, block edges, a random spread."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    rng = np.random.default_rng(seed)
    toks = set()
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if b == a:
            continue
        for off in (0, 1, 2, block_size - 1, block_size, block_size + 1, 2 * block_size + 5):
            if a + off < b:
                toks.add(a + off)
        for off in (1, 2, block_size // 2):
            if b - off >= a:
                toks.add(b - off)
        L = b - a
        for x in rng.integers(0, L, size=max(1, n_random * L // max(int(cu[-1]), 1))):
            toks.add(a + int(x))
    return np.array(sorted(toks), dtype=np.int64)


def max_abs(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        d = np.abs(np.where(both_inf, 0.0, a - b))
    return float(np.nan_to_num(d, nan=np.inf).max()) if d.size else 0.0


def bf16_half_ulp(x):
    """Half the spacing of bfloat16 numbers at |x| (0 at x = 0)."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(x > 0, x, 1.0)))
    return np.where(x > 0, np.exp2(e - 8), 0.0)


def o_excess(o_gpu, o_ref):
    """max over elements of |O_gpu - O_ref| - half_ulp_bf16(O_ref): the kernel's error
    beyond the unavoidable rounding of the exact answer to the bf16 output format."""
    a = np.asarray(o_gpu, dtype=np.float64)
    b = np.asarray(o_ref, dtype=np.float64)
    return float((np.abs(a - b) - bf16_half_ulp(b)).max()) if a.size else 0.0


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a))


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
