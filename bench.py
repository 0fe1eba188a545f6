#!/usr/bin/env python
"""Benchmark of NSA selected-block attention (forward + backward) on B200.

One step = the whole path on one batch: forward (index inversion, tensor-core tile
kernel, log-sum-exp merge) then backward (inversion, D = rowsum(dO * O), tile
kernel, dQ merge, dK/dV reduction) of the headline workload: one sequence of
T = 65536 tokens, 16 query heads over 4 KV heads (group 4), head_dim 128,
block 64, top-16 blocks per (token, KV head), bf16 inputs ~ N(0, 1).

`value` is useful TFLOP/s: 4 * d * (keys attended after the causal mask) per query
head per token for the forward, 2.5x that for the backward, summed over all ranks
and divided by the device time of K steps (CUDA events, max over ranks).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own independent problem (weak scaling, no data
collective).  `--impl reference` times the fp64 CPU oracle on a bounded sample of
the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import nsa_inputs as ni  # noqa: E402

METRIC = "selected-attn fwd/bwd TFLOP/s and ms at T=64k; % of B200 bf16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- work

def attended_keys(cu_seqlens, block_idx, block_size, window=0):
    """Keys each (token, KV head) row attends after the causal mask and, for window > 0,
    the sliding window of that many keys (counting only)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T, hkv, topk = block_idx.shape
    out = np.zeros((T, hkv), dtype=np.int64)
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if b == a:
            continue
        i = np.arange(b - a, dtype=np.int64)
        qb = (i // block_size)[:, None, None]
        x = block_idx[a:b].astype(np.int64)
        x = np.sort(np.where((x >= 0) & (x <= qb), x, -1), axis=2)
        first = np.ones_like(x, dtype=bool)
        first[:, :, 1:] = x[:, :, 1:] != x[:, :, :-1]
        keep = first & (x >= 0)
        if window <= 0:
            full = (keep & (x < qb)).sum(axis=2)
            diag = (keep & (x == qb)).sum(axis=2)
            out[a:b] = full * block_size + diag * ((i % block_size) + 1)[:, None]
        else:
            ii = i[:, None, None]
            lo = np.maximum(x * block_size, ii - window + 1)
            hi = np.minimum((x + 1) * block_size - 1, ii)
            out[a:b] = np.where(keep, np.maximum(hi - lo + 1, 0), 0).sum(axis=2)
    return out


def useful_flops(p: ni.Problem, window=0):
    keys = attended_keys(p.cu_seqlens, p.block_idx, p.block_size, window)
    G = p.hq // p.hkv
    fwd = 4.0 * p.head_dim * float(keys.sum()) * G
    return fwd, 2.5 * fwd


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks, clk):
    """The bf16 tensor peak a kernel timed in this run is measured against: the burst
    figure while the sampled SM clock held its maximum (a short timed region), the
    power-capped sustained figure once the median clock fell below 97 % of it."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    sm, smax = (clk or {}).get("sm_mhz"), (clk or {}).get("sm_max_mhz")
    if sm and smax and sm < 0.97 * smax:
        return "bf16_tflops_sustained", sustained
    return "bf16_tflops", burst


def unique_bytes(p: ni.Problem, tdt=None):
    """Bytes every forward / backward call must move at least once (each input read and
    each output written once): forward Q, K, V, block_idx, cu_seqlens in, O and LSE
    out; backward Q, K, V, O, dO, LSE, block_idx, cu_seqlens in, dQ, dK, dV out."""
    e = 2   # bf16 / fp16
    q = p.T * p.hq * p.head_dim * e
    kv = p.T * p.hkv * p.head_dim * e
    idx = p.block_idx.size * 4 + p.cu_seqlens.size * 4
    lse = p.hq * p.T * 4
    fwd = q + 2 * kv + idx + q + lse
    bwd = (q + 2 * kv + q + q + lse + idx) + (q + 2 * kv)
    return float(fwd), float(bwd)


def l2_note(p: ni.Problem, tdt=None):
    q = p.T * p.hq * p.head_dim * 2
    part = p.block_idx.size * (p.hq // p.hkv) * (p.head_dim * 2 + 8)
    return (f"inputs larger than L2 (Q {q / 1e6:.0f} MB, forward partials up to "
            f"{part / 1e9:.2f} GB); no flush")


# source file of each kernel whose DRAM traffic the committed ncu summary records
KERNEL_SOURCES = {"k_fwd_tiles": "fwd.cu", "k_bwd_tiles": "bwd.cu", "k_merge": "merge.cu",
                  "k_dq_merge": "merge.cu"}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the kernel's source file and the shared headers."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_attention_selected_b200", "csrc")
    for f in (KERNEL_SOURCES[kernel], "nsa_common.cuh", "nsa_kernels.h"):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, launch_units: float):
    """DRAM bytes per launch from the committed ncu summary, if it matches the sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        d = json.load(open(path))
    except Exception:
        return None
    k = d.get("kernels", {}).get(kernel)
    if not k or kernel not in KERNEL_SOURCES or k.get("source_hash") != kernel_source_hash(kernel):
        return None
    # stored per unit of work (useful FLOP) so that a smaller capture scales
    return float(k["dram_bytes_per_useful_flop"]) * launch_units


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples during the timed region (read-only queries)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="nsa_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].lower().startswith("active")})
        loaded = [s for s, r in zip(sm, rows) if num(r[3]) and num(r[3]) > 200] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(pw) if pw else None,
                "samples": len(rows), "reasons": reasons}


# ------------------------------------------------------------------------- our arm

def rank_spec(workload: str, rank: int) -> dict:
    """Problem of one rank: the workload's shapes, its own seed (independent problems)."""
    spec = dict(ni.WORKLOADS[workload])
    spec["seed"] = spec["seed"] + 1000 * rank
    return spec


def max_over_ranks(x: float, dist, device) -> float:
    """The largest of every rank's value (the job time of a weak-scaling step)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, step_flops: float, steps: int, elapsed_ms: float) -> float:
    """Useful TFLOP/s of the whole job: every rank's steps over the slowest rank's time."""
    return world * step_flops * steps / (elapsed_ms * 1e-3) / 1e12


def run_ours(args, rank, world, local_rank, dist):
    import torch
    import block_sparse_attention_selected_b200 as nsa
    from block_sparse_attention_selected_b200 import build as nsa_build

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    nsa_build.build()
    lib = nsa.load_library()

    spec = rank_spec(args.workload, rank)
    p = ni.make_problem(name=args.workload, head_dim=128, with_dout=True, **spec)
    W = args.window
    if W > 0:   # the sliding branch: every block the window reaches, then the window mask
        p.block_idx = ni.band_block_idx(p.cu_seqlens, p.hkv, p.topk, p.block_size, W)
    fwd_flops, bwd_flops = useful_flops(p, W)
    step_flops = fwd_flops + bwd_flops
    T, hq, hkv, d, topk, bs, nseq = p.T, p.hq, p.hkv, 128, p.topk, p.block_size, p.nseq

    tdt = torch.float16 if args.dtype == "fp16" else torch.bfloat16
    f16_flag = nsa.NSA_F16 if args.dtype == "fp16" else 0
    bf = lambda a: torch.from_numpy(a).to(tdt).pin_memory()
    h_q, h_k, h_v, h_do = bf(p.q), bf(p.k), bf(p.v), bf(p.dout)
    h_cu = torch.from_numpy(p.cu_seqlens).pin_memory()
    h_bi = torch.from_numpy(np.ascontiguousarray(p.block_idx)).pin_memory()
    q, k, v, do = (x.to(dev) for x in (h_q, h_k, h_v, h_do))
    cu, bi = h_cu.to(dev), h_bi.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((hq, T), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = nsa.nsa_sel_attn_workspace_size(T, nseq, hq, hkv, d, topk, bs, True)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes_ptr = nsa._ptr
    scale = p.scale
    import ctypes
    n_fwd = ctypes.c_int(0)
    n_bwd = ctypes.c_int(0)

    def ev_array(evs):
        # torch creates the CUDA event lazily: record once so that the handle exists
        for e in evs:
            e.record(stream)
        torch.cuda.synchronize()
        handles = [e.cuda_event for e in evs]
        assert all(handles), "CUDA events were not created"
        arr = (ctypes.c_void_p * len(evs))(*handles)
        return ctypes.cast(arr, ctypes.c_void_p), arr

    def step(fwd_ev=None, bwd_ev=None, q_=q, k_=k, v_=v, do_=do, cu_=cu, bi_=bi):
        rc = lib.nsa_sel_attn_fwd_ex(
            sp(q_), sp(k_), sp(v_), sp(cu_), nseq, T, hq, hkv, d, sp(bi_), topk, bs, scale,
            sp(out), sp(lse), sp(ws), ws_bytes, ctypes.c_void_p(stream.cuda_stream), f16_flag, W,
            fwd_ev, 4 if fwd_ev is not None else 0, ctypes.byref(n_fwd))
        if rc:
            raise RuntimeError(f"forward failed: {rc}")
        # the backward reuses the index inversion the forward left in the shared workspace
        rc = lib.nsa_sel_attn_bwd_ex(
            sp(q_), sp(k_), sp(v_), sp(out), sp(lse), sp(do_), sp(cu_), nseq, T, hq, hkv, d,
            sp(bi_), topk, bs, scale, sp(dq), sp(dk), sp(dv), sp(ws), ws_bytes,
            ctypes.c_void_p(stream.cuda_stream), nsa.NSA_BWD_REUSE_INDEX | f16_flag, W, bwd_ev,
            6 if bwd_ev is not None else 0, ctypes.byref(n_bwd))
        if rc:
            raise RuntimeError(f"backward failed: {rc}")

    def step_on(strm, ins, outs):
        # one forward + backward on stream `strm` with explicit device buffers
        q_, k_, v_, do_, cu_, bi_ = ins
        o_, l_, dq_, dk_, dv_ = outs
        h = ctypes.c_void_p(strm.cuda_stream)
        rc = lib.nsa_sel_attn_fwd_ex(
            sp(q_), sp(k_), sp(v_), sp(cu_), nseq, T, hq, hkv, d, sp(bi_), topk, bs, scale,
            sp(o_), sp(l_), sp(ws), ws_bytes, h, f16_flag, W, None, 0, None)
        if rc:
            raise RuntimeError(f"forward failed: {rc}")
        rc = lib.nsa_sel_attn_bwd_ex(
            sp(q_), sp(k_), sp(v_), sp(o_), sp(l_), sp(do_), sp(cu_), nseq, T, hq, hkv, d,
            sp(bi_), topk, bs, scale, sp(dq_), sp(dk_), sp(dv_), sp(ws), ws_bytes, h,
            nsa.NSA_BWD_REUSE_INDEX | f16_flag, W, None, 0, None)
        if rc:
            raise RuntimeError(f"backward failed: {rc}")

    def barrier():
        if dist is not None:
            dist.barrier()


    # warm-up
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = nsa.nsa_sel_check_status(ws)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {st}")

    K = args.steps
    fevs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    bevs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
    farr_keep = [ev_array(e) for e in fevs]
    barr_keep = [ev_array(e) for e in bevs]
    farr = [a for a, _ in farr_keep]
    barr = [a for a, _ in barr_keep]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local_rank)
    clocks = ClockSampler(gpu_id)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    for i in range(K):
        step(farr[i], barr[i])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), dist, dev)
    if nsa.nsa_sel_check_status(ws) != 0:
        raise RuntimeError("device status error in the timed region")
    ms_step = elapsed_ms / K
    value = job_tflops(world, step_flops, K, elapsed_ms)

    def avg(evs, a, b):
        return statistics.mean(e[a].elapsed_time(e[b]) for e in evs)

    phase = {
        "fwd_ms": avg(fevs, 0, 3), "fwd_invert_ms": avg(fevs, 0, 1),
        "fwd_tiles_ms": avg(fevs, 1, 2), "fwd_merge_ms": avg(fevs, 2, 3),
        "bwd_ms": avg(bevs, 0, 5), "bwd_invert_ms": avg(bevs, 0, 1),
        "bwd_delta_ms": avg(bevs, 1, 2), "bwd_tiles_ms": avg(bevs, 2, 3),
        "bwd_dq_merge_ms": avg(bevs, 3, 4), "bwd_dkdv_reduce_ms": avg(bevs, 4, 5),
    }
    peaks, peak_src = load_peaks()
    peak_name, tc_peak = tensor_peak(peaks, clk)
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    if phase["bwd_tiles_ms"] >= phase["fwd_tiles_ms"]:
        dom, dom_ms, dom_flops = "k_bwd_tiles", phase["bwd_tiles_ms"], bwd_flops
    else:
        dom, dom_ms, dom_flops = "k_fwd_tiles", phase["fwd_tiles_ms"], fwd_flops
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 2),
                "peak": tc_peak, "unit": "TFLOP/s", "frac": round(achieved / tc_peak, 4),
                "peak_source": f"{peak_name} of {peak_src}",
                "traffic": profiled_traffic(dom, dom_flops)}
    # whole-call roofline fractions: max(FLOPs / tensor peak, unique bytes / HBM peak)
    # over the call's measured time (inversion and merges included)
    fb, bb = unique_bytes(p, tdt)
    fwd_floor = max(fwd_flops / (tc_peak * 1e12), fb / (hbm_peak * 1e9)) * 1e3
    bwd_floor = max(bwd_flops / (tc_peak * 1e12), bb / (hbm_peak * 1e9)) * 1e3
    roofline["fwd_frac"] = round(fwd_floor / phase["fwd_ms"], 4)
    roofline["bwd_frac"] = round(bwd_floor / phase["bwd_ms"], 4)
    roofline["step_frac"] = round((fwd_floor + bwd_floor) / ms_step, 4)
    roofline["call_fracs"] = ("max(useful FLOPs / tensor peak, unique bytes / HBM copy peak "
                              f"{hbm_peak:.0f} GB/s) / measured call ms")
    fwd_tiles_tflops = fwd_flops / (phase["fwd_tiles_ms"] * 1e-3) / 1e12
    bwd_tiles_tflops = bwd_flops / (phase["bwd_tiles_ms"] * 1e-3) / 1e12
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))

    # end to end through the C ABI with host buffers: H2D inputs, fwd+bwd, D2H outputs
    e2e = None
    if not args.no_e2e:
        h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        h_dq = torch.empty(dq.shape, dtype=dq.dtype).pin_memory()
        h_dk = torch.empty(dk.shape, dtype=dk.dtype).pin_memory()
        h_dv = torch.empty(dv.shape, dtype=dv.dtype).pin_memory()
        h_in = [h_q, h_k, h_v, h_do, h_cu, h_bi]
        h_res = [h_out, h_lse, h_dq, h_dk, h_dv]
        h2d = sum(x.numel() * x.element_size() for x in h_in)
        d2h = sum(x.numel() * x.element_size() for x in h_res)
        Ke = max(2, min(K, 5))
        # A pipeline of three streams: the input copies of step k + 1 and the output
        # copies of step k - 1 overlap the compute of step k (device inputs and outputs
        # double-buffered).  Every step's H2D and D2H lie inside the timed region, which
        # runs from the first input copy to the last output copy.
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        d_in = [[torch.empty_like(x) for x in (q, k, v, do, cu, bi)] for _ in range(2)]
        d_out = [[torch.empty_like(x) for x in (out, lse, dq, dk, dv)] for _ in range(2)]

        def run_e2e(nsteps, start_ev=None, end_ev=None):
            comp_done, out_done = [], []
            if start_ev is not None:
                start_ev.record(s_in)
            for kk in range(nsteps):
                bb = kk % 2
                in_ready = torch.cuda.Event()
                with torch.cuda.stream(s_in):
                    if kk >= 2:                         # compute kk - 2 has read buffer bb
                        s_in.wait_event(comp_done[kk - 2])
                    for dst, src in zip(d_in[bb], h_in):
                        dst.copy_(src, non_blocking=True)
                    in_ready.record(s_in)
                stream.wait_event(in_ready)
                if kk >= 2:                             # outputs of kk - 2 copied out
                    stream.wait_event(out_done[kk - 2])
                step_on(stream, d_in[bb], d_out[bb])
                cd = torch.cuda.Event()
                cd.record(stream)
                comp_done.append(cd)
                od = torch.cuda.Event()
                with torch.cuda.stream(s_out):
                    s_out.wait_event(cd)
                    for dst, src in zip(h_res, d_out[bb]):
                        dst.copy_(src, non_blocking=True)
                    od.record(s_out)
                out_done.append(od)
            if end_ev is not None:
                end_ev.record(s_out)

        run_e2e(2)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        run_e2e(Ke, a, b)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(a.elapsed_time(b), dist, dev)
        e2e = {"value": round(job_tflops(world, step_flops, Ke, e_ms), 3), "unit": UNIT,
               "ms_per_step": round(e_ms / Ke, 3), "steps": Ke,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "overlap": "H2D of step k+1 and D2H of step k-1 run on their own streams "
                          "during the compute of step k (double-buffered device buffers)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, tokens=args.cpu_tokens, window=W)

    launches = K * (n_fwd.value + n_bwd.value)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": args.dtype,
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V/dO; index rule init+local+random earlier)"
                if W == 0 else "synthetic (seeded N(0,1) bf16 Q/K/V/dO; sliding-branch index: "
                               "every block the window reaches)",
        "config": {"workload": args.workload, "total_tokens": T, "num_seqs": nseq, "hq": hq,
                   "hkv": hkv, "group": hq // hkv, "head_dim": d, "block_size": bs, "topk": topk,
                   "window_size": W,
                   "parallelism": f"independent problem per rank x{world}",
                   "l2": l2_note(p, tdt)},
        "fwd_ms": round(phase["fwd_ms"], 4), "bwd_ms": round(phase["bwd_ms"], 4),
        "fwd_tflops": round(fwd_flops / (phase["fwd_ms"] * 1e-3) / 1e12, 2),
        "bwd_tflops": round(bwd_flops / (phase["bwd_ms"] * 1e-3) / 1e12, 2),
        "fwd_pct_of_bf16_peak": round(100 * fwd_flops / (phase["fwd_ms"] * 1e-3) / 1e12 / burst, 2),
        "fwd_pct_of_bf16_sustained_peak": round(
            100 * fwd_flops / (phase["fwd_ms"] * 1e-3) / 1e12 / sustained, 2),
        "fwd_tiles_tflops": round(fwd_tiles_tflops, 2),
        "bwd_tiles_tflops": round(bwd_tiles_tflops, 2),
        "phases_ms": {k2: round(v2, 4) for k2, v2 in phase.items()},
        "useful_tflop_per_step": round(step_flops / 1e12, 4),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
        "gpu_launches": launches,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return line


# ------------------------------------------------- the selection step and BSFA

def run_next_path(args):
    """One GPU, CUDA events: the block-selection step (compression, block scores,
    top-k) or threshold-pruned block attention on the workload's shapes; one JSON line."""
    import torch
    import block_sparse_attention_selected_b200 as nsa
    from block_sparse_attention_selected_b200 import build as nsa_build
    nsa_build.build()
    dev = torch.device("cuda", 0)
    spec = dict(ni.WORKLOADS[args.workload])
    p = ni.make_problem(name=args.workload, head_dim=128, with_dout=False, **spec)
    bf = lambda a: torch.from_numpy(a).to(dev).to(torch.bfloat16)
    q, k, v = bf(p.q), bf(p.k), bf(p.v)
    cu = torch.from_numpy(p.cu_seqlens).to(dev)
    T, hq, hkv, bs, d = p.T, p.hq, p.hkv, p.block_size, 128
    lens = np.diff(p.cu_seqlens.astype(np.int64))
    i = np.concatenate([np.arange(L) for L in lens]) if T else np.zeros(0, np.int64)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    times = []
    if args.path == "select":
        nb = int(max((L + bs - 1) // bs for L in lens))
        visible = np.where(i >= 31, (i - 31) // 16 + 1, 0)            # compressed keys seen
        useful = 2.0 * d * float(visible.sum()) * hq                    # one Q Kc^T
        issued = 2 * useful                                             # two passes
        ws = nsa.get_workspace(int(nsa.load_library().nsa_sel_block_scores_workspace_size(p.nseq)), dev)

        def step():
            evs[0].record()
            kc, _, cu_cmp = nsa.nsa_sel_compress_kv(k, v, cu)
            evs[1].record()
            sc = nsa.nsa_sel_block_scores(q, kc, cu, cu_cmp, bs, nb, p.scale, workspace=ws)
            evs[2].record()
            nsa.nsa_sel_select_topk(sc, cu, bs, p.topk, 1, 2, workspace=ws)
            evs[3].record()
        names = ("compress_ms", "scores_ms", "topk_ms")
    else:
        tau = torch.full((hq,), float(args.tau), dtype=torch.float32, device=dev)
        causal = (i + 1).astype(np.float64)
        useful = 2.0 * d * float(causal.sum()) * hq                     # exact scores (one pass)
        issued = 3 * useful                                             # two S passes + PV on every block

        def step():
            evs[0].record()
            nsa.nsa_sel_bsfa_fwd(q, k, v, cu, tau, p.scale)
            evs[1].record()
            evs[2].record()
            evs[3].record()
        names = ("bsfa_ms",)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        step()
        torch.cuda.synchronize()
        times.append([evs[a].elapsed_time(evs[a + 1]) for a in range(len(names))])
    status = nsa.nsa_sel_check_status()
    t = np.median(np.asarray(times), axis=0)
    kernel_ms = float(t[1] if args.path == "select" else t[0])
    line = {"metric": f"{args.path} step ms and TFLOP/s", "path": args.path,
            "value": round(float(t.sum()), 4), "unit": "ms", "higher_is_better": False,
            "steps": args.steps, "warmup": max(args.warmup, 3), "status": int(status),
            "config": {"workload": args.workload, "total_tokens": T, "hq": hq, "hkv": hkv,
                       "block_size": bs, "topk": p.topk,
                       **({"tau": float(args.tau)} if args.path == "bsfa" else {})},
            "phases_ms": {n: round(float(x), 4) for n, x in zip(names, t)},
            "useful_tflops": round(useful / (kernel_ms * 1e-3) / 1e12, 2),
            "issued_tflops": round(issued / (kernel_ms * 1e-3) / 1e12, 2)}
    print(json.dumps(line), flush=True)
    return line


# ----------------------------------------------------------------- oracle baselines

def oracle_sample(workload: str, tokens: int, window: int = 0):
    spec = dict(ni.WORKLOADS[workload])
    spec["lengths"] = [min(tokens, sum(spec["lengths"]))]
    p = ni.make_problem(name=workload + f"_prefix{tokens}", head_dim=128, **spec)
    if window > 0:
        p.block_idx = ni.band_block_idx(p.cu_seqlens, p.hkv, p.topk, p.block_size, window)
    return p


def time_oracle_step(p, nthreads, window=0):
    import oracle
    t = time.perf_counter()
    oracle.fwd(p.q, p.k, p.v, p.cu_seqlens, p.block_idx, p.block_size, p.scale, window=window,
               nthreads=nthreads)
    oracle.bwd(p.q, p.k, p.v, p.dout, p.cu_seqlens, p.block_idx, p.block_size, p.scale,
               window=window, nthreads=nthreads)
    return time.perf_counter() - t


def cpu_baseline(workload: str, tokens: int, window: int = 0):
    cores = len(os.sched_getaffinity(0))
    p = oracle_sample(workload, tokens, window)
    f, b = useful_flops(p, window)
    dt = time_oracle_step(p, cores, window)
    return {"value": round((f + b) / dt / 1e12, 6), "unit": UNIT, "cores": cores,
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"first {p.T} tokens (all {p.hq} heads) of the workload, forward + full "
                      f"backward in fp64; useful FLOPs by the same formula"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    cores = len(os.sched_getaffinity(0))
    p = oracle_sample(args.workload, args.ref_tokens, args.window)
    f, b = useful_flops(p, args.window)
    for _ in range(args.warmup):
        time_oracle_step(p, cores, args.window)
    times = [time_oracle_step(p, cores, args.window) for _ in range(args.steps)]
    total = sum(times)
    value = (f + b) * len(times) / total / 1e12
    sample = (f"first {p.T} tokens (all {p.hq} heads) of the workload per step, forward + full "
              f"backward in fp64")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1000 * total / len(times), 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "sample_tokens": p.T,
                       "window_size": args.window},
            "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample,
                             "value": round(value, 6), "unit": UNIT},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return line


# ---------------------------------------------------------------------------- main

def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=ni.HEADLINE, choices=sorted(ni.WORKLOADS))
    ap.add_argument("--dtype", choices=["bf16", "fp16"], default="bf16",
                    help="element type of q, k, v, dO and the outputs (fp32 arithmetic)")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding window of this many keys (0: none); the index becomes the "
                         "sliding branch's: every block the window reaches")
    ap.add_argument("--path", choices=["attn", "select", "bsfa"], default="attn",
                    help="attn: the selected attention step (the default line); select: the "
                         "block-selection step; bsfa: threshold-pruned block attention")
    ap.add_argument("--tau", type=float, default=2.0, help="BSFA threshold of every head")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=2048)
    ap.add_argument("--ref-tokens", type=int, default=1024)
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return 0
    if args.path != "attn":
        if rank == 0:
            run_next_path(args)
        return 0
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    try:
        run_ours(args, rank, world, local_rank, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
