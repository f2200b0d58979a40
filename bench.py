#!/usr/bin/env python
"""Benchmark of ReHyAt's chunked hybrid attention forward on B200.

Workload (one step = one full forward through the C ABI): the 5 s, 480x832
Wan2.1-1.3B-shaped layer -- latent 21x30x52 (N = 32760 tokens), batch 2,
12 heads, D = 128, D' = 128, T_c = 3, T_o = 1, bidirectional, bf16 q/k/v
drawn by rehyat_inputs (seed 2), fp32 output.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints ONE JSON line (rank 0).  Device time is measured with CUDA events on
the stream the kernels run on, with an L2 flush before every timed step
(outside the events: a 256 MB write, then a 256 MB read of a second buffer,
so that no input and no dirty line is left in L2), max over ranks.  ``--impl reference`` times the fp64
CPU oracle on a bounded sample instead (rank 0 only).

Multi-GPU: every rank runs the same workload on its own GPU (replicas; the
path has no exchange step), so ``value`` = all ranks' tokens / max time.  The
extra measurements beside the step (comparator, fp8, backward, general
feature maps, streaming) run at N = 1 only.
"""
from __future__ import annotations

import argparse
import datetime as _dt
import hashlib
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "wan_480x832_bidir"
METRIC = "hybrid-attn fwd tokens/s & TFLOP/s (% BF16 tensor peak), 1 B200, 21x30x52 latent"
L2_FLUSH_BYTES = 256 << 20
KERNELS_PER_STEP = 4  # weight images, per-slice state, chunk scan, attention
EXTRAS = ("full_softmax", "fp8_qk", "phi_backward", "full_backward", "general_phi", "streaming")
E2E_HEADS_PER_SLAB = 2


class L2Flush:
    """Empties L2 (126 MB on B200) between timed steps: a 256 MB write evicts
    every input, and a 256 MB read of a second buffer then evicts the write's
    dirty lines, so the timed kernels neither find their inputs in L2 nor pay
    for writing back data that is not theirs."""

    def __init__(self, torch, dev):
        n = L2_FLUSH_BYTES // 4
        self.wbuf = torch.empty(n, dtype=torch.float32, device=dev)
        self.rbuf = torch.zeros(n, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)
        self.torch = torch

    def __call__(self):
        self.wbuf.zero_()
        self.torch.sum(self.rbuf, dim=0, out=self.sink)


# --------------------------------------------------------------- workload
def workload_desc(p):
    return (f"{WORKLOAD}: B={p.batch}, heads={p.heads}, latent {p.T}x{p.Hs}x{p.Ws} "
            f"(N={p.N}), D={p.D}, D'={p.Dp}, T_c={p.Tc}, T_o={p.To}, "
            f"{'causal' if p.causal else 'bidirectional'}, bf16 q/k/v, fp32 y")


def algorithmic_work(B, h, T, HW, D, Dp, Tc, To, causal):
    """Method FLOPs / bytes (not the dense-attention work they avoid).

    softmax: 4*D per (query, window key) pair (q.k and p.v);
    phi_q, phi_k: 2*D*Dp per token each;  state: 2*Dp*D (+Dp) per token;
    readout: 2*Dp*D (+2*Dp) per token.  All per (batch, head)."""
    N = T * HW
    pairs = 0
    for t in range(-(-T // Tc)):
        first, end = t * Tc, min(T, (t + 1) * Tc)
        w = max(first - To, 0)
        pairs += (end - first) * HW * (end - w) * HW
    bh = B * h
    f_soft = 4.0 * D * pairs * bh
    f_phi = 2.0 * N * D * Dp * bh
    f_state = (2.0 * N * Dp * D + N * Dp) * bh
    f_read = (2.0 * N * Dp * D + 2.0 * N * Dp) * bh
    return dict(
        attn_flops=f_soft + f_phi + f_read,       # attention kernel (K3)
        state_flops=f_phi + f_state,              # per-slice state kernel (K1)
        total_flops=f_soft + 2 * f_phi + f_state + f_read,
        exps=float(pairs * bh),
        # K1 minimal HBM traffic: read k, v (bf16); write per-slice states (fp32)
        state_bytes=float(bh * (2 * N * D * 2 + T * (Dp * D + Dp) * 4)),
        # whole op minimal traffic: q, k, v in, y out (fp32), states out
        io_bytes=float(bh * (3 * N * D * 2 + N * D * 4 + T * (Dp * D + Dp) * 4)),
        full_softmax_flops=4.0 * D * N * N * bh,
    )


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", 0.0)),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                    source="fallback")


def kernel_source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_traffic(kernel_key, sha):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[kernel_key]
        if e.get("source_sha") == sha:
            return float(e["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        pass
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.lines = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self, t0, t1):
        rows = []
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = _dt.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]), parts[4:]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05] or rows[-3:]
        if not inside:
            return None
        sm = sorted(r[1] for r in inside)
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = set()
        for r in inside:
            for name, val in zip(names[1:], r[3][1:]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": inside[0][2],
                "reasons": sorted(reasons), "samples": len(inside)}


# ------------------------------------------------------------- CPU oracle
def host_info():
    """CPU model and the BLAS library the oracle's numpy runs on (for the
    CPU baseline's record); fields it cannot read are left out."""
    info = {}
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    info["cpu"] = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        from threadpoolctl import threadpool_info
        libs = [f"{i.get('internal_api', '?')} {i.get('version', '')}".strip()
                for i in threadpool_info() if i.get("user_api") == "blas"]
        if libs:
            info["blas"] = ", ".join(sorted(set(libs)))
    except Exception:
        pass
    return info


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def plan_oracle_sample(p, budget_s):
    """Size a bounded sample of the workload for the fp64 oracle (factored
    form, as it stands): time one chunk of one (batch, head) pair once, then
    take as many chunks (or whole pairs) as fit in ``budget_s`` seconds."""
    from oracle import rehyat_oracle as orc
    nch = -(-p.T // p.Tc)
    t0 = time.perf_counter()
    orc.run_problem(p, heads_subset=[0], chunks_subset=[nch // 2])
    one_chunk = time.perf_counter() - t0
    if one_chunk * nch > budget_s:
        return dict(heads=1, chunks=max(1, min(nch, int(budget_s / max(one_chunk, 1e-6)))))
    BH = p.batch * p.heads
    return dict(heads=max(1, min(BH, int(budget_s / (one_chunk * nch)))), chunks=nch)


def run_oracle_sample(p, plan, start_head=0):
    from oracle import rehyat_oracle as orc
    nch = -(-p.T // p.Tc)
    BH = p.batch * p.heads
    heads = [(start_head + i) % BH for i in range(plan["heads"])]
    chunks = list(range(plan["chunks"]))
    t0 = time.perf_counter()
    orc.run_problem(p, heads_subset=heads, chunks_subset=None if len(chunks) == nch else chunks)
    dt = time.perf_counter() - t0
    rows = sum((min(p.T, (c + 1) * p.Tc) - c * p.Tc) * p.HW for c in chunks)
    # tokens of the metric count all heads of a token: rows * pairs / heads
    token_equiv = rows * len(heads) / p.heads
    return dict(seconds=dt, token_equiv=token_equiv,
                sample=f"{len(heads)} of {BH} (batch, head) pairs x chunks "
                       f"{chunks[0]}..{chunks[-1]} of {nch} ({rows} query rows per pair)")


# ------------------------------------------------------ extra measurements
def measure_full_softmax(rh, q, k, v, y, flush, stream, calls=3):
    """Plain softmax over all N keys on the same tensors (the dense
    comparator the ReHyAt note measures against), device time per call."""
    import torch
    B, H, N, D = q.shape
    p = rh.make_params(batch=B, heads=H, T=1, Hs=1, Ws=N, D=D, Dp=32, Tc=1, To=0, causal=0,
                       in_dtype=rh.BF16, out_dtype=rh.F32)
    sh = stream.cuda_stream
    call = lambda: rh.rehyat_softmax_attn_fwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                              y.data_ptr(), sh)
    if call():
        raise RuntimeError("rehyat_softmax_attn_fwd failed")
    times = []
    for _ in range(calls):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return {"ms": sum(times) / len(times), "calls": calls,
            "what": "rehyat_softmax_attn_fwd on the same q, k, v (all N keys per query)"}


FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # CUDA-core fp32 FMA peak at 1965 MHz


def measure_phi_backward(rh, p, q, k, v, Wq, bq, Wk, bk, flush, stream, calls=3):
    """rehyat_phi_bwd on the bench workload: forward with the denominators
    exported (nS, nL), an upstream gradient from a seeded torch generator,
    then device time per backward call (fp32 CUDA-core kernels)."""
    import torch
    B, H, N, D = q.shape
    dev = q.device
    params = rh.make_params(batch=B, heads=H, T=p.T, Hs=p.Hs, Ws=p.Ws, D=D, Dp=p.Dp, Tc=p.Tc,
                            To=p.To, causal=p.causal, in_dtype=rh.BF16, out_dtype=rh.F32)
    sh = stream.cuda_stream
    phi = rh.RehyatPhi(Wq.data_ptr(), bq.data_ptr(), Wk.data_ptr(), bk.data_ptr())
    y = torch.empty(B, H, N, D, device=dev)
    nS = torch.empty(B, H, N, device=dev)
    nL = torch.empty(B, H, N, device=dev)
    dbg = rh.RehyatDebug(None, nS.data_ptr(), None, None, nL.data_ptr())
    ws = torch.empty(max(rh.rehyat_workspace_bytes(params), rh.rehyat_phi_bwd_workspace_bytes(params)),
                     dtype=torch.uint8, device=dev)
    if rh.rehyat_hybrid_attn_fwd(params, q.data_ptr(), k.data_ptr(), v.data_ptr(), phi,
                                 y.data_ptr(), ws.data_ptr(), ws.numel(), dbg, sh):
        raise RuntimeError("rehyat_hybrid_attn_fwd failed")
    den = nS + nL
    g = torch.Generator(device=dev).manual_seed(5)
    dy = torch.randn(B, H, N, D, generator=g, device=dev)
    grads = {n: torch.empty_like(t) for n, t in (("dWq", Wq), ("dbq", bq), ("dWk", Wk), ("dbk", bk))}
    gs = rh.RehyatPhiGrad(*(grads[n].data_ptr() for n in ("dWq", "dbq", "dWk", "dbk")))
    # The second form runs on the forward's workspace (REHYAT_FLAG_FWD_STATE):
    # the backward reads the forward's linear-set state instead of repeating
    # the state pass.  Every plain call rewrites that state with the same bits.
    reuse = rh.make_params(batch=B, heads=H, T=p.T, Hs=p.Hs, Ws=p.Ws, D=D, Dp=p.Dp, Tc=p.Tc,
                           To=p.To, causal=p.causal, in_dtype=rh.BF16, out_dtype=rh.F32,
                           flags=rh.FLAG_FWD_STATE)
    call = lambda prm: rh.rehyat_phi_bwd(prm, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         y.data_ptr(), dy.data_ptr(), den.data_ptr(), phi, gs,
                                         ws.data_ptr(), ws.numel(), sh)
    if call(params):
        raise RuntimeError("rehyat_phi_bwd failed")
    ref = {n: t.clone() for n, t in grads.items()}
    if call(reuse):
        raise RuntimeError("rehyat_phi_bwd (forward's state) failed")
    same = all(torch.equal(ref[n], grads[n]) for n in grads)

    def timed(prm):
        times = []
        for _ in range(calls):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call(prm)
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        return sum(times) / len(times)
    ms = timed(params)
    ms_fs = timed(reuse)
    # Algorithmic FLOPs of the backward proper (per token and (b,h): u_q, dphi_q,
    # dW_q, G_t on the q side, u_k, dphi_k, dW_k on the k side, each 2*D*D'),
    # plus the state pass it repeats (phi_k and phi_k^T v: 4*D*D').
    flops = B * H * N * D * p.Dp * 2.0 * (7 + 2)
    flops_fs = B * H * N * D * p.Dp * 2.0 * 7
    del y, nS, nL, ws, dy
    tflops = flops / (ms / 1e3) / 1e12
    if D == 128 and p.Dp == 128:  # q and k passes on tcgen05 (bf16 operands)
        peaks = load_peaks()
        roof = {"bound": "tensor", "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": tflops / peaks["bf16_tflops"],
                "peak_source": "measured bf16 burst (MEASURED_PEAKS.json)"}
    else:
        roof = {"bound": "alu", "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s",
                "frac": tflops / FP32_ALU_TFLOPS,
                "peak_source": "148 SMs x 128 fp32 FMA lanes x 2 x 1965 MHz"}
    tf_fs = flops_fs / (ms_fs / 1e3) / 1e12
    return {"ms": ms, "calls": calls, "tflops": tflops, "roofline": roof,
            "with_forward_state": {"ms": ms_fs, "tflops": tf_fs,
                                   "frac": tf_fs / roof["peak"], "bitwise_equal": same},
            "what": "rehyat_phi_bwd (dW_q, db_q, dW_k, db_k) on the bench workload, bf16 "
                    "q/k/v, fp32 y, dy, den; `ms` includes its state pass, "
                    "`with_forward_state` reuses the forward's (REHYAT_FLAG_FWD_STATE)"}


def measure_full_backward(rh, p, q, k, v, Wq, bq, Wk, bk, flush, stream, calls=3):
    """rehyat_hybrid_attn_bwd on the bench workload: forward with c and the
    denominators exported, an upstream gradient from a seeded torch generator,
    then device time per full backward call (dq, dk, dv and the feature-map
    gradients, its state pass included)."""
    import torch
    B, H, N, D = q.shape
    dev = q.device
    params = rh.make_params(batch=B, heads=H, T=p.T, Hs=p.Hs, Ws=p.Ws, D=D, Dp=p.Dp, Tc=p.Tc,
                            To=p.To, causal=p.causal, in_dtype=rh.BF16, out_dtype=rh.F32)
    sh = stream.cuda_stream
    phi = rh.RehyatPhi(Wq.data_ptr(), bq.data_ptr(), Wk.data_ptr(), bk.data_ptr())
    y = torch.empty(B, H, N, D, device=dev)
    c = torch.empty(B, H, N, device=dev)
    nS = torch.empty(B, H, N, device=dev)
    nL = torch.empty(B, H, N, device=dev)
    dbg = rh.RehyatDebug(None, nS.data_ptr(), c.data_ptr(), None, nL.data_ptr())
    ws = torch.empty(max(rh.rehyat_workspace_bytes(params),
                         rh.rehyat_hybrid_attn_bwd_workspace_bytes(params)),
                     dtype=torch.uint8, device=dev)
    if rh.rehyat_hybrid_attn_fwd(params, q.data_ptr(), k.data_ptr(), v.data_ptr(), phi,
                                 y.data_ptr(), ws.data_ptr(), ws.numel(), dbg, sh):
        raise RuntimeError("rehyat_hybrid_attn_fwd failed")
    den = nS + nL
    del nS, nL
    g = torch.Generator(device=dev).manual_seed(6)
    dy = torch.randn(B, H, N, D, generator=g, device=dev)
    out = {n: torch.empty(B, H, N, D, device=dev) for n in ("dq", "dk", "dv")}
    grads = {n: torch.empty_like(t) for n, t in (("dWq", Wq), ("dbq", bq), ("dWk", Wk), ("dbk", bk))}
    gs = rh.RehyatPhiGrad(*(grads[n].data_ptr() for n in ("dWq", "dbq", "dWk", "dbk")))
    reuse = rh.make_params(batch=B, heads=H, T=p.T, Hs=p.Hs, Ws=p.Ws, D=D, Dp=p.Dp, Tc=p.Tc,
                           To=p.To, causal=p.causal, in_dtype=rh.BF16, out_dtype=rh.F32,
                           flags=rh.FLAG_FWD_STATE)
    call = lambda prm: rh.rehyat_hybrid_attn_bwd(
        prm, q.data_ptr(), k.data_ptr(), v.data_ptr(), phi, y.data_ptr(), dy.data_ptr(),
        c.data_ptr(), den.data_ptr(), out["dq"].data_ptr(), out["dk"].data_ptr(),
        out["dv"].data_ptr(), gs, ws.data_ptr(), ws.numel(), sh)
    if call(params):
        raise RuntimeError("rehyat_hybrid_attn_bwd failed")

    def timed(prm):
        times = []
        for _ in range(calls):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call(prm)
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        return sum(times) / len(times)
    ms = timed(params)
    ms_fs = timed(reuse)
    # Algorithmic FLOPs: the softmax branch's backward, 10 D per (query,
    # window key) pair (S and dP recomputed, dV, dQ, dK), plus the feature-map
    # part (the phi-gradient extra's count) and the linear branch's token
    # gradients (dq, dk through phi: 2 D D' each; dv: 2 D D').
    w = algorithmic_work(B, H, p.T, p.Hs * p.Ws, D, p.Dp, p.Tc, p.To, p.causal)
    pairs = w["exps"]  # (query, window key) pairs over every (b, h)
    flops = 10.0 * D * pairs + B * H * N * D * p.Dp * 2.0 * (7 + 2 + 3)
    del y, c, den, ws, dy, out
    tflops = flops / (ms / 1e3) / 1e12
    peaks = load_peaks()
    return {"ms": ms, "calls": calls, "tflops": tflops,
            "roofline": {"bound": "tensor", "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tflops / peaks["bf16_tflops"],
                         "peak_source": "measured bf16 burst (MEASURED_PEAKS.json)",
                         "work_per_call": f"{flops:.4e} FLOP"},
            "with_forward_state": {"ms": ms_fs},
            "what": "rehyat_hybrid_attn_bwd (dq, dk, dv, dW_q, db_q, dW_k, db_k) on the bench "
                    "workload, bf16 q/k/v, fp32 y, dy, c, den; `ms` includes its state pass, "
                    "`with_forward_state` reuses the forward's (REHYAT_FLAG_FWD_STATE)"}


def measure_general_phi(rh, p, q, k, v, flush, stream, calls=3):
    """General feature maps on the bench workload: the per-head 2-layer MLP
    (hidden width 3D, P = 2 parts) for q and for k, then the forward with the
    maps given (rehyat_hybrid_attn_fwd_phi).  Device time per call of each,
    with the maps in bf16 (REHYAT_FLAG_PHI_BF16) and in fp32."""
    import torch
    B, H, N, D = q.shape
    dev = q.device
    Dp, Dh = p.Dp, 3 * D
    g = torch.Generator(device=dev).manual_seed(6)
    Wa = torch.randn(H, D, Dh, generator=g, device=dev) / D ** 0.5
    ba = 0.1 * torch.randn(H, Dh, generator=g, device=dev)
    Wb = 0.5 * torch.randn(H, Dh, Dp, generator=g, device=dev) / Dh ** 0.5
    bb = 0.05 * torch.randn(H, Dp, generator=g, device=dev)
    sh = stream.cuda_stream
    mlp = rh.RehyatPhiMlp(Wa.data_ptr(), ba.data_ptr(), Wb.data_ptr(), bb.data_ptr(), Dh, 2)
    y = torch.empty(B, H, N, D, device=dev)
    peaks = load_peaks()

    def timed(fn):
        times = []
        for _ in range(calls):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        return sum(times) / len(times)

    def run(phi_dtype):
        flags = rh.FLAG_PHI_BF16 if phi_dtype == torch.bfloat16 else 0
        params = rh.make_params(batch=B, heads=H, T=p.T, Hs=p.Hs, Ws=p.Ws, D=D, Dp=Dp, Tc=p.Tc,
                                To=p.To, causal=p.causal, in_dtype=rh.BF16, out_dtype=rh.F32,
                                flags=flags)
        pq = torch.empty(B, H, N, Dp, device=dev, dtype=phi_dtype)
        pk = torch.empty(B, H, N, Dp, device=dev, dtype=phi_dtype)
        ws = torch.empty(rh.rehyat_workspace_bytes(params), dtype=torch.uint8, device=dev)
        mlp_bytes = rh.rehyat_feature_map_mlp_workspace_bytes(params, mlp, q.data_ptr(),
                                                              pq.data_ptr())
        mws = torch.empty(max(mlp_bytes, 16), dtype=torch.uint8, device=dev)
        feat = lambda: (rh.rehyat_feature_map_mlp(params, q.data_ptr(), mlp, pq.data_ptr(),
                                                  mws.data_ptr(), mlp_bytes, sh) or
                        rh.rehyat_feature_map_mlp(params, k.data_ptr(), mlp, pk.data_ptr(),
                                                  mws.data_ptr(), mlp_bytes, sh))
        fwd = lambda: rh.rehyat_hybrid_attn_fwd_phi(params, q.data_ptr(), k.data_ptr(),
                                                    v.data_ptr(), pq.data_ptr(), pk.data_ptr(),
                                                    y.data_ptr(), ws.data_ptr(), ws.numel(),
                                                    None, sh)
        if feat() or fwd():
            raise RuntimeError("general feature map path failed")
        feat_ms, fwd_ms = timed(feat), timed(fwd)
        del pq, pk, ws, mws
        return feat_ms, fwd_ms, mlp_bytes > 0

    feat_ms, fwd_ms, tensor_cores = run(torch.bfloat16)
    feat32_ms, fwd32_ms, _ = run(torch.float32)
    feat_flops = 2 * B * H * N * (2.0 * D * Dh + 2.0 * Dh * Dp)  # q and k
    # Algorithmic bytes: x in (bf16) and phi out (bf16) for q and k; the
    # weights (2.4 MB of images) are negligible.
    feat_bytes = 2 * B * H * N * (D * 2 + Dp * 2)
    tflops = feat_flops / (feat_ms / 1e3) / 1e12
    gbs = feat_bytes / (feat_ms / 1e3) / 1e9
    del y
    out = {"feature_maps_ms": feat_ms,
           "feature_maps_path": "tensor cores (bf16 operands)" if tensor_cores
           else "fp32 CUDA cores",
           "feature_maps_dtype": "bf16",
           "feature_maps_tflops": tflops,
           "feature_maps_gbs": gbs,
           "forward_phi_given_ms": fwd_ms,
           "forward_phi_given_tokens_per_s": B * N / (fwd_ms / 1e3),
           "maps_plus_forward_ms": feat_ms + fwd_ms,
           "fp32_maps": {"feature_maps_ms": feat32_ms, "forward_phi_given_ms": fwd32_ms,
                         "maps_plus_forward_ms": feat32_ms + fwd32_ms},
           "what": "rehyat_feature_map_mlp for q and k (hidden 3D = 384, P = 2), then "
                   "rehyat_hybrid_attn_fwd_phi (tensor-core path) on the bench workload; "
                   "maps in bf16 (REHYAT_FLAG_PHI_BF16), and in fp32 under fp32_maps"}
    if tensor_cores:
        out["feature_maps_frac_bf16_peak"] = tflops / peaks["bf16_tflops"]
        out["feature_maps_frac_hbm"] = gbs / peaks["hbm_gbs"]
    else:
        out["feature_maps_alu_frac"] = tflops / FP32_ALU_TFLOPS
    return out


def measure_fp8_qk(rh, p, q, k, v, phi, flush, stream, calls=5):
    """The fp8 softmax-branch variant (REHYAT_FLAG_FP8_QK) on the bench
    layer: the same step (state stage, then the E4M3 copies of q and k and the
    attention kernel with q.k^T on kind::f8f6f4), device time per stage."""
    import torch
    B, H, N, D = q.shape
    params = rh.make_params(batch=B, heads=H, T=p.T, Hs=p.Hs, Ws=p.Ws, D=D, Dp=p.Dp, Tc=p.Tc,
                            To=p.To, causal=p.causal, in_dtype=rh.BF16, out_dtype=rh.F32,
                            flags=rh.FLAG_FP8_QK)
    nbytes = rh.rehyat_workspace_bytes(params)
    if nbytes == 0:
        return {"unavailable": "REHYAT_FLAG_FP8_QK not supported for this layer"}
    ws = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    y = torch.empty(B, H, N, D, device=q.device)
    sh = stream.cuda_stream

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        st = rh.rehyat_fwd_state(params, k.data_ptr(), v.data_ptr(), phi, ws.data_ptr(), nbytes,
                                 sh)
        if evs:
            evs[1].record(stream)
        st = st or rh.rehyat_fwd_attn(params, q.data_ptr(), k.data_ptr(), v.data_ptr(), phi,
                                      y.data_ptr(), ws.data_ptr(), nbytes, None, sh)
        if evs:
            evs[2].record(stream)
        if st:
            raise rh.RehyatError(st, "fp8 forward")

    for _ in range(3):
        flush()
        step()
    torch.cuda.synchronize()
    t_step, t_attn = [], []
    for _ in range(calls):
        flush()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        step(evs)
        torch.cuda.synchronize()
        t_step.append(evs[0].elapsed_time(evs[2]))
        t_attn.append(evs[1].elapsed_time(evs[2]))
    w = algorithmic_work(B, H, p.T, p.HW, D, p.Dp, p.Tc, p.To, p.causal)
    peaks = load_peaks()
    ms, attn_ms = sum(t_step) / calls, sum(t_attn) / calls
    del ws, y
    return {"ms_per_step": ms, "attention_stage_ms": attn_ms,
            "tokens_per_s": B * N / (ms / 1e3),
            "attention_tflops": w["attn_flops"] / (attn_ms / 1e3) / 1e12,
            "attention_frac_bf16_peak": w["attn_flops"] / (attn_ms / 1e3) / 1e12
            / peaks["bf16_tflops"],
            "what": "REHYAT_FLAG_FP8_QK: q.k^T from E4M3 copies of q, k (kind::f8f6f4), P.V "
                    "and the linear branch bf16; the attention stage includes the E4M3 "
                    "conversion kernel"}


def measure_streaming(rh, dev, flush, stream):
    """Chunk-wise RNN over 81 slices of 30x52 (27 steps of T_c = 3, T_o = 1,
    12 heads, D = D' = 128): per-step device time, steady-state tokens/s,
    free device memory before and after the 27 steps."""
    import torch
    g = torch.Generator(device=dev).manual_seed(3)
    H, HW, D, Dp, Tc, To, T = 12, 30 * 52, 128, 128, 3, 1, 81
    rows = Tc * HW

    def draw(shape, scale=1.0):
        return torch.randn(shape, generator=g, device=dev, dtype=torch.float32) * scale

    s = 0.5 + 1.5 * torch.rand((3, H, 1, 1), generator=g, device=dev)
    q = (draw((1, H, T * HW, D)) * s[0]).to(torch.bfloat16)
    k = (draw((1, H, T * HW, D)) * s[1]).to(torch.bfloat16)
    v = (draw((1, H, T * HW, D)) * s[2]).to(torch.bfloat16)
    Wq, Wk = draw((H, 2, D, Dp // 2), 0.1), draw((H, 2, D, Dp // 2), 0.1)
    bq, bk = draw((H, 2, Dp // 2), 0.1), draw((H, 2, Dp // 2), 0.1)
    chunks = [tuple(x[:, :, i * rows:(i + 1) * rows].contiguous() for x in (q, k, v))
              for i in range(T // Tc)]
    del q, k, v
    st = rh.StreamingState(batch=1, heads=H, Hs=30, Ws=52, D=D, Dp=Dp, Tc=Tc, To=To, Wq=Wq,
                           bq=bq, Wk=Wk, bk=bk, in_dtype=torch.bfloat16, device=dev)
    out = torch.empty(1, H, rows, D, device=dev)
    for c in chunks[:3]:  # warm-up
        st.step(*c, out=out)
    st.reset()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(dev)[0]
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in chunks]
    for (e0, e1), c in zip(evs, chunks):
        e0.record(stream)
        st.step(*c, out=out)
        e1.record(stream)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info(dev)[0]
    ms = [e0.elapsed_time(e1) for e0, e1 in evs]
    steady = sorted(ms[2:])[len(ms[2:]) // 2]
    y_eager = out.clone()

    # The same 27 steps as one captured step replayed per chunk (the chunk is
    # copied into fixed input buffers first; the copies, 43 MB per step, are
    # inside the timing).
    st.reset()
    qb, kb, vb = (torch.empty_like(x) for x in chunks[0])
    outg = torch.empty_like(out)
    graph = st.capture_step(qb, kb, vb, outg)
    gevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in chunks]
    for (e0, e1), c in zip(gevs, chunks):
        e0.record(stream)
        qb.copy_(c[0])
        kb.copy_(c[1])
        vb.copy_(c[2])
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    gms = [e0.elapsed_time(e1) for e0, e1 in gevs]
    gsteady = sorted(gms[2:])[len(gms[2:]) // 2]
    same = bool(torch.equal(outg, y_eager))
    del graph

    # All 27 steps captured as one graph over the chunks in place (no input
    # copies), replayed once: the whole stream with a single graph launch.
    st.reset()
    outs = torch.empty_like(out)
    seq = st.capture_steps(chunks, outs)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    seq.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    seq_ms = e0.elapsed_time(e1)
    seq_same = bool(torch.equal(outs, y_eager))
    del seq
    return {"workload": "81 slices of 30x52, 12 heads, D=D'=128, T_c=3, T_o=1, bf16, "
                        "27 rehyat_chunk_step calls (inputs from a seeded torch generator)",
            "steps": len(ms), "ms_per_step_median_steady": steady,
            "ms_first_steps": ms[:3], "tokens_per_s_steady": rows / (steady / 1e3),
            "graph_ms_per_step_median_steady": gsteady,
            "graph_tokens_per_s_steady": rows / (gsteady / 1e3),
            "graph_last_chunk_bitwise_equal_to_eager": same,
            "sequence_graph_ms_per_step": seq_ms / len(chunks),
            "sequence_graph_tokens_per_s": rows * len(chunks) / (seq_ms / 1e3),
            "sequence_graph_last_chunk_bitwise_equal_to_eager": seq_same,
            "free_bytes_before": free0, "free_bytes_after": free1,
            "device_memory_constant": free0 == free1}


def run_sweep(args):
    """T_c in {1,2,3,5,7} x T_o in {0,1,2} x D' in {64,128,256} x {bidirectional,
    causal} on the 21x30x52 latent (batch 2, 12 heads, D = 128, bf16), q and k
    low-rank (rank 8) plus N(0, 0.3^2) noise, v ~ N(0,1), from a seeded torch
    generator.  One JSON line per point: step time, tokens/s and the
    attention kernel's fraction of the measured bf16 peak."""
    import torch
    import linear_attention_video_chunked_b200 as rh
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev).manual_seed(4)
    B, H, T, Hs, Ws, D = 2, 12, 21, 30, 52, 128
    HW, N = Hs * Ws, T * Hs * Ws
    G = torch.randn(H, 8, D, generator=g, device=dev) / math.sqrt(8.0)

    def lowrank():
        u = torch.randn(B, H, N, 8, generator=g, device=dev)
        x = torch.einsum("bhnr,hrd->bhnd", u, G)
        return (x + 0.3 * torch.randn(B, H, N, D, generator=g, device=dev)).to(torch.bfloat16)

    q, k = lowrank(), lowrank()
    v = torch.randn(B, H, N, D, generator=g, device=dev).to(torch.bfloat16)
    y = torch.empty(B, H, N, D, device=dev)
    flush = L2Flush(torch, dev)
    peaks = load_peaks()
    stream = torch.cuda.current_stream()
    csrc = sorted(os.path.join("linear_attention_video_chunked_b200", "csrc", f)
                  for f in os.listdir(os.path.join(ROOT, "linear_attention_video_chunked_b200",
                                                   "csrc"))
                  if f.endswith((".cu", ".cuh", ".h")))
    print(json.dumps({"sweep": "21x30x52", "header": True,
                      "source_sha": kernel_source_sha(csrc + ["include/rehyat.h"]),
                      "peak_bf16_tflops": peaks["bf16_tflops"], "peak_source": peaks["source"],
                      "peak_hbm_gbs": peaks["hbm_gbs"]}), flush=True)
    points = [(Dp, causal, Tc, To, 0) for Dp in (64, 128, 256) for causal in (0, 1)
              for Tc in (1, 2, 3, 5, 7) for To in (0, 1, 2)]
    # The fp8 q.k^T variant at D' = 128, both forms.
    points += [(128, causal, Tc, To, rh.FLAG_FP8_QK) for causal in (0, 1)
               for Tc in (1, 2, 3, 5, 7) for To in (0, 1, 2)]
    phis = {}
    for Dp in (64, 128, 256):
        Wq, Wk = (0.1 * torch.randn(H, 2, D, Dp // 2, generator=g, device=dev) for _ in range(2))
        bq, bk = (0.1 * torch.randn(H, 2, Dp // 2, generator=g, device=dev) for _ in range(2))
        phis[Dp] = (rh.RehyatPhi(Wq.data_ptr(), bq.data_ptr(), Wk.data_ptr(), bk.data_ptr()),
                    (Wq, bq, Wk, bk))
    for Dp, causal, Tc, To, flags in points:
        phi = phis[Dp][0]
        p = rh.make_params(batch=B, heads=H, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc,
                           To=To, causal=causal, in_dtype=rh.BF16, out_dtype=rh.F32,
                           flags=flags)
        nbytes = rh.rehyat_workspace_bytes(p)
        if nbytes == 0:
            continue
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)

        def call(evs=None):
            if evs:
                evs[0].record(stream)
            rh.rehyat_fwd_state(p, k.data_ptr(), v.data_ptr(), phi, ws.data_ptr(),
                                nbytes, stream.cuda_stream)
            if evs:
                evs[1].record(stream)
            st = rh.rehyat_fwd_attn(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), phi,
                                    y.data_ptr(), ws.data_ptr(), nbytes, None,
                                    stream.cuda_stream)
            if st:
                raise rh.RehyatError(st, "rehyat_fwd_attn")
            if evs:
                evs[2].record(stream)

        for _ in range(3):
            call()
        times = []
        for _ in range(max(3, args.steps // 6)):
            flush()
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            call(evs)
            torch.cuda.synchronize()
            times.append((evs[0].elapsed_time(evs[2]), evs[1].elapsed_time(evs[2])))
        step_ms = sum(t[0] for t in times) / len(times)
        attn_ms = sum(t[1] for t in times) / len(times)
        w = algorithmic_work(B, H, T, HW, D, Dp, Tc, To, causal)
        attn_tf = w["attn_flops"] / (attn_ms / 1e3) / 1e12
        state_gbs = w["state_bytes"] / ((step_ms - attn_ms) / 1e3) / 1e9
        print(json.dumps({
            "sweep": "21x30x52", "Tc": Tc, "To": To, "Dp": Dp,
            "form": "causal" if causal else "bidirectional",
            "qk": "fp8 e4m3" if flags else "bf16",
            "attn_kernel": "tensor-core two-tile" if rh.rehyat_attn_path(p) == 1
            else "CUDA-core",
            "ms_per_step": step_ms, "tokens_per_s": B * N / (step_ms / 1e3),
            "state_ms": step_ms - attn_ms, "state_frac_hbm": state_gbs / peaks["hbm_gbs"],
            "attn_ms": attn_ms, "attn_tflops": attn_tf,
            "attn_frac_bf16_peak": attn_tf / peaks["bf16_tflops"],
            "total_tflop": w["total_flops"] / 1e12,
            "full_softmax_over_hybrid_flops": w["full_softmax_flops"] / w["total_flops"],
        }), flush=True)
        del ws
    return 0


# ------------------------------------------------------------ multi-rank
def max_over_ranks(ms, dist=None, device=None):
    """Device time of the slowest rank (every rank calls this, in order)."""
    if dist is None:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, tokens_per_step, steps, max_ms):
    """Whole-job tokens/s: every rank runs the same workload (replicas), so
    the job processed world * tokens_per_step * steps tokens in max_ms."""
    return world * tokens_per_step * steps / (max_ms / 1e3)


# --------------------------------------------------------------- main arms
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    from rehyat_inputs import config_problem
    p = config_problem(WORKLOAD)
    per_step = max(0.5, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    plan = plan_oracle_sample(p, per_step)
    for i in range(args.warmup):
        run_oracle_sample(p, plan, start_head=i)
    total_s, total_tok, samples = 0.0, 0.0, []
    for i in range(args.steps):
        r = run_oracle_sample(p, plan, start_head=args.warmup + i)
        total_s += r["seconds"]
        total_tok += r["token_equiv"]
        samples.append(r["sample"])
    value = total_tok / total_s
    cores = blas_threads()
    w = algorithmic_work(p.batch, p.heads, p.T, p.HW, p.D, p.Dp, p.Tc, p.To, p.causal)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(p), "global_batch": p.batch, "seq_len": p.N,
                   "parallelism": "none (host cores)"},
        "tflops": w["total_flops"] / (p.batch * p.N) * value / 1e12,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: {samples[0]}", "host": host_info()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_gpu(args, world, rank, local):
    import numpy as np
    import torch

    import linear_attention_video_chunked_b200 as rh
    from rehyat_inputs import config_problem

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=_dt.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    rh.lib()

    # --batch/--heads draw a smaller case of the same layer (profiler captures).
    p = config_problem(WORKLOAD, **{k: v for k, v in (("batch", args.batch), ("heads", args.heads))
                                    if v is not None})
    B, H, N, D = p.q.shape
    T, HW, Dp = p.T, p.HW, p.Dp
    bf = torch.bfloat16
    tt = lambda a, d: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dtype=d)
    q, k, v = tt(p.q, bf), tt(p.k, bf), tt(p.v, bf)
    Wq, bq, Wk, bk = (tt(a, torch.float32) for a in (p.Wq, p.bq, p.Wk, p.bk))
    y = torch.empty(B, H, N, D, device=dev, dtype=torch.float32)
    params = rh.make_params(batch=B, heads=H, T=T, Hs=p.Hs, Ws=p.Ws, D=D, Dp=Dp, Tc=p.Tc,
                            To=p.To, causal=p.causal, in_dtype=rh.BF16, out_dtype=rh.F32)
    ws_bytes = rh.rehyat_workspace_bytes(params)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    phi = rh.RehyatPhi(Wq.data_ptr(), bq.data_ptr(), Wk.data_ptr(), bk.data_ptr())
    flush = L2Flush(torch, dev)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        st = rh.rehyat_fwd_state(params, k.data_ptr(), v.data_ptr(), phi, ws.data_ptr(),
                                 ws_bytes, sh)
        if st:
            raise rh.RehyatError(st, "rehyat_fwd_state")
        if evs:
            evs[1].record(stream)
        st = rh.rehyat_fwd_attn(params, q.data_ptr(), k.data_ptr(), v.data_ptr(), phi,
                                y.data_ptr(), ws.data_ptr(), ws_bytes, None, sh)
        if st:
            raise rh.RehyatError(st, "rehyat_fwd_attn")
        if evs:
            evs[2].record(stream)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    time.sleep(0.3)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_host0 = time.time()
    for i in range(args.steps):
        flush()
        step(events[i])
    torch.cuda.synchronize()
    t_host1 = time.time()
    if dist:
        dist.barrier()
    clocks.stop()
    step_ms = [e[0].elapsed_time(e[2]) for e in events]
    state_ms = [e[0].elapsed_time(e[1]) for e in events]
    attn_ms = [e[1].elapsed_time(e[2]) for e in events]
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    ms_per_step = total_ms / args.steps
    tokens_per_step = B * N
    value = job_throughput(world, tokens_per_step, args.steps, total_ms)

    # End to end through the C ABI with host buffers: rehyat_hybrid_attn_fwd_host
    # uploads q, k, v from pinned host memory and downloads y, slabs of two
    # heads in flight on three streams; every copy is inside the timed region.
    qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
    yh = torch.empty(B, H, N, D, dtype=torch.float32).pin_memory()
    per_slab = E2E_HEADS_PER_SLAB
    hws_bytes = rh.rehyat_host_workspace_bytes(params, per_slab)
    hws = torch.empty(hws_bytes, dtype=torch.uint8, device=dev)
    e2e_steps = max(1, min(args.steps, 10))

    def e2e_step():
        st = rh.rehyat_hybrid_attn_fwd_host(params, qh.data_ptr(), kh.data_ptr(), vh.data_ptr(),
                                            phi, yh.data_ptr(), per_slab, hws.data_ptr(),
                                            hws_bytes, sh)
        if st:
            raise rh.RehyatError(st, "rehyat_hybrid_attn_fwd_host")

    e2e_step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    if dist:
        dist.barrier()
    e2e_value = job_throughput(world, tokens_per_step, e2e_steps, e2e_ms)
    h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh))
    d2h = yh.numel() * yh.element_size()
    del qh, kh, vh, yh, hws

    extra = {}
    want = set(EXTRAS if args.extras is None else args.extras.split(","))
    if args.no_extras or world > 1:
        # The extras describe one GPU; with replicas they would only hold every
        # GPU of the job longer.
        want = set()
    if "full_softmax" in want:
        with torch.cuda.nvtx.range("full_softmax"):
            extra["full_softmax"] = measure_full_softmax(rh, q, k, v, y, flush, stream)
    del y, ws
    torch.cuda.empty_cache()
    if "fp8_qk" in want:
        with torch.cuda.nvtx.range("fp8_qk"):
            extra["fp8_qk"] = measure_fp8_qk(rh, p, q, k, v, phi, flush, stream)
        torch.cuda.empty_cache()
    if "phi_backward" in want:
        with torch.cuda.nvtx.range("phi_backward"):
            extra["phi_backward"] = measure_phi_backward(rh, p, q, k, v, Wq, bq, Wk, bk, flush,
                                                         stream)
        torch.cuda.empty_cache()
    if "full_backward" in want:
        with torch.cuda.nvtx.range("full_backward"):
            extra["full_backward"] = measure_full_backward(rh, p, q, k, v, Wq, bq, Wk, bk,
                                                           flush, stream)
        torch.cuda.empty_cache()
    if "general_phi" in want:
        with torch.cuda.nvtx.range("general_phi"):
            extra["general_phi"] = measure_general_phi(rh, p, q, k, v, flush, stream)
    del q, k, v
    torch.cuda.empty_cache()
    if "streaming" in want:
        with torch.cuda.nvtx.range("streaming"):
            extra["streaming"] = measure_streaming(rh, dev, flush, stream)

    if rank != 0:
        if dist:
            dist.destroy_process_group()
        return 0

    w = algorithmic_work(B, H, T, HW, D, Dp, p.Tc, p.To, p.causal)
    peaks = load_peaks()
    attn_avg_s = sum(attn_ms) / len(attn_ms) / 1e3
    state_avg_s = sum(state_ms) / len(state_ms) / 1e3
    achieved_tf = w["attn_flops"] / attn_avg_s / 1e12
    sha = kernel_source_sha(["linear_attention_video_chunked_b200/csrc/tc_kernels.cu",
                             "linear_attention_video_chunked_b200/csrc/tc_common.cuh"])
    roofline = {"kernel": "attention (window softmax + phi_q readout + joint norm)",
                "bound": "tensor", "achieved": achieved_tf, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved_tf / peaks["bf16_tflops"],
                "traffic": load_traffic("attn", sha),
                "peak_source": f"{peaks['source']} bf16 burst (MEASURED_PEAKS.json)"
                if peaks["source"] == "measured" else "fallback 1.59 PFLOP/s",
                "work_per_launch": f"{w['attn_flops']:.4e} FLOP "
                                   f"(4*D per query-key pair in the window + phi_q + readout)"}
    if peaks.get("bf16_tflops_sustained"):
        # The same kernel against the seconds-long power-capped GEMM figure.
        roofline["frac_of_sustained"] = achieved_tf / peaks["bf16_tflops_sustained"]
        roofline["peak_sustained"] = peaks["bf16_tflops_sustained"]
    state_gbs = w["state_bytes"] / state_avg_s / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload_desc(p), "global_batch": B * world, "seq_len": N,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "flushed before every timed step, outside the events: 256 MB write, then 256 MB read of a second buffer"},
        "tflops": w["total_flops"] / (ms_per_step / 1e3) / 1e12 * world,
        "pct_bf16_peak": w["total_flops"] / (ms_per_step / 1e3) / 1e12 / peaks["bf16_tflops"],
        "stages_ms": {"state (per-slice + scan)": sum(state_ms) / len(state_ms),
                      "attention": sum(attn_ms) / len(attn_ms)},
        "ms_per_step_median": sorted(step_ms)[len(step_ms) // 2],
        "ms_per_step_min": min(step_ms),
        "state_stage_hbm": {"achieved": state_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": state_gbs / peaks["hbm_gbs"],
                            "bytes_per_launch": w["state_bytes"]},
        "roofline": roofline,
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "api": "rehyat_hybrid_attn_fwd_host (C ABI), pinned host q, k, v, y",
                "heads_per_slab": E2E_HEADS_PER_SLAB},
        "clocks": clocks.summary(t_host0, t_host1),
    }
    line.update(extra)
    if "full_softmax" in extra:
        fs = extra["full_softmax"]
        fs["tflops"] = w["full_softmax_flops"] / (fs["ms"] / 1e3) / 1e12
        fs["frac_bf16_peak"] = fs["tflops"] / peaks["bf16_tflops"]
        fs["hybrid_speedup"] = fs["ms"] / ms_per_step
    if world == 1 and not args.no_cpu_baseline:
        r = run_oracle_sample(p, plan_oracle_sample(p, args.cpu_budget))
        cv = r["token_equiv"] / r["seconds"]
        line["cpu_baseline"] = {"value": cv, "unit": "tokens/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": r["sample"],
                                "seconds": r["seconds"], "host": host_info()}
    print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["own", "reference"], default="own")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of fp64 oracle work for the CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="T_c/T_o/D'/form sweep on the 21x30x52 latent, one JSON line per point")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the measurements beside the step (comparator, backward, "
                         "general feature maps, streaming)")
    ap.add_argument("--extras", default=None,
                    help="comma-separated subset of " + ",".join(EXTRAS))
    ap.add_argument("--batch", type=int, default=None,
                    help="batch of a smaller case of the layer (default: the workload's 2)")
    ap.add_argument("--heads", type=int, default=None,
                    help="heads of a smaller case of the layer (default: the workload's 12)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    world, rank, local = dist_setup()
    if args.sweep:
        return run_sweep(args) if rank == 0 else 0
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_gpu(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
