#!/usr/bin/env python
"""BitLinear W1.58A8 benchmark on B200.

Workload (default, "decode"): one token (M=1) through the seven BitLinear
projections (q, k, v, o, gate, up, down) of each of the 30 layers of the
BitNet b1.58 2B4T shapes: 210 full BitLinear forwards per step (RMSNorm with
U(0.5,1.5) gain, per-token int8 quantisation, ternary matmul, rescale, bf16
output), each with its own input as the decode workload specifies, 521 MB of
distinct packed weights, more than the 126 MB L2, so every step streams them
from HBM.  Inputs: x ~ N(0,1) with 0.1% outliers x20; weights
absmean-ternarised from N(0, 0.02) masters.  tokens/s = M / step time.

The headline runs the 210 forwards as one batched call (a quantise launch and
one GEMV launch); the line also reports one batched call per layer, one call
per projection, and the GEMV kernel alone.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs its own replica (the path has no exchange step)
and the reported value is the tokens of all ranks / the slowest rank's time.
Prints one JSON line on rank 0.
"""
import argparse
import ctypes
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "BitLinear W1.58A8 tokens/s; % roofline (GEMV HBM GB/s, GEMM int8 TOPS)"
DECODE_KERNEL_SOURCES = ("common.cuh", "decode.cuh")
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--layers", type=int, default=30)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU work budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-skinny", action="store_true",
                    help="skip the batched-decode (8/32/64 tokens) measurements")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the M=4096 prefill measurement reported beside the headline")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup(timeout_s=300):
    """One process per GPU under torchrun (NCCL); the same plumbing runs on
    CPU-only hosts over gloo (tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            torch.distributed.init_process_group(
                "nccl", timeout=datetime.timedelta(seconds=timeout_s),
                device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group(
                "gloo", timeout=datetime.timedelta(seconds=timeout_s))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v, world):
    """The slowest rank's value (every rank calls this, in the same order)."""
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, ms):
    """Whole-job units per second: every rank processed units_per_rank in at
    most ms (the max over ranks of the device-timed region)."""
    return world * units_per_rank / (ms / 1000.0)


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting"}

    def __init__(self, index):
        self.samples = []
        self.reasons = 0
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # reported, never fatal
            self.err = repr(e)

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self.stop_flag.is_set():
            self._sample()
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.stop_flag = threading.Event()
            self._sample()
            self.th = threading.Thread(target=self._run, daemon=True)
            self.th.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._sample()
            self.stop_flag.set()
            self.th.join()

    def result(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        reasons = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# the decode workload
# ---------------------------------------------------------------------------
def token_work_units(WL, layers):
    """Per-projection MAC counts (work units) of one token through all layers."""
    return sum(p.N * p.K for p in WL.PROJECTIONS) * layers


class DecodeWorkload:
    """The 210 problems of one token, plus CUDA graphs of the ways to run them."""

    def __init__(self, layers, M=1):
        import ternary_weight_bitlinear_b200 as B
        from ternary_weight_bitlinear_b200 import workloads as WL
        self.B, self.WL, self.M, self.layers = B, WL, M, layers
        dev = torch.device("cuda")
        specs = [(l, p) for l in range(layers) for p in WL.PROJECTIONS]
        x_elems = sum(M * p.K for _, p in specs)
        y_elems = sum(M * p.N for _, p in specs)
        self.x_dev = torch.empty(x_elems, dtype=torch.bfloat16, device=dev)
        self.y_dev = torch.empty(y_elems, dtype=torch.bfloat16, device=dev)
        self.x_host = torch.empty(x_elems, dtype=torch.bfloat16).pin_memory()
        self.y_host = torch.empty(y_elems, dtype=torch.bfloat16).pin_memory()
        self.problems = []
        gains = {}
        xo = yo = 0
        self.weight_bytes = 0
        for l, p in specs:
            W = torch.from_numpy(WL.master_weights(p.N, p.K, WL.master_seed(l, p.name))).to(dev)
            P, beta = B.bitlinear_pack(W)
            del W
            c = WL.config2_projection(l, p.name, M)
            xv = torch.from_numpy(c["x"].reshape(-1).view(np.int16)).view(torch.bfloat16)
            self.x_host[xo:xo + xv.numel()].copy_(xv)
            key = (l, p.K)
            if key not in gains:
                gains[key] = torch.from_numpy(c["gain"].view(np.int16)).view(torch.bfloat16).to(dev)
            self.problems.append(dict(
                layer=l, name=p.name, x=self.x_dev[xo:xo + M * p.K].view(M, p.K), P=P, beta=float(beta.item()),
                gain=gains[key], y=self.y_dev[yo:yo + M * p.N].view(M, p.N), K=p.K, N=p.N))
            self.weight_bytes += P.numel()
            xo += M * p.K
            yo += M * p.N
        self.x_dev.copy_(self.x_host)
        torch.cuda.synchronize()
        # a second set of input/output buffers, so that the end-to-end run can
        # copy one step's inputs in and the previous step's outputs out while a
        # step computes
        self.x_dev2 = torch.empty_like(self.x_dev)
        self.y_dev2 = torch.empty_like(self.y_dev)
        self.problems2 = []
        xo = yo = 0
        for q in self.problems:
            q2 = dict(q)
            q2["x"] = self.x_dev2[xo:xo + M * q["K"]].view(M, q["K"])
            q2["y"] = self.y_dev2[yo:yo + M * q["N"]].view(M, q["N"])
            self.problems2.append(q2)
            xo += M * q["K"]
            yo += M * q["N"]
        # algorithmic bytes of one step: packed weights + x + gain + y
        self.step_bytes = self.weight_bytes + 2 * (x_elems + sum(p["K"] for p in self.problems)
                                                   + y_elems)
        self.h2d_bytes = 2 * x_elems
        self.d2h_bytes = 2 * y_elems
        eps = WL.RMS_EPS
        # one batch per layer (the headline), one batch per token, one call per projection
        self.layer_batches = []
        for l in range(layers):
            items = [q for q in self.problems if q["layer"] == l]
            arr = B.make_batch(items)
            ws = torch.empty(max(16, B.bitlinear_forward_batch_workspace_size(arr, M)),
                             dtype=torch.uint8, device=dev)
            self.layer_batches.append((arr, ws, items))
        self.token_batch = B.make_batch(self.problems)
        self.token_batch2 = B.make_batch(self.problems2)
        self.token_ws = torch.empty(B.bitlinear_forward_batch_workspace_size(self.token_batch, M),
                                    dtype=torch.uint8, device=dev)
        for q in self.problems:
            q["ws"] = torch.empty(B.bitlinear_forward_workspace_size(M, q["K"], q["N"]),
                                  dtype=torch.uint8, device=dev)
        # pre-quantised codes for timing the GEMV kernel alone
        self.gemv_batches = []
        self.gemv_bytes = 0
        for l in range(layers):
            items = []
            for q in self.problems:
                if q["layer"] != l:
                    continue
                qq, sx, rs = B.bitlinear_act_quant(q["x"], q["gain"], eps)
                items.append(dict(q=qq, s_x=sx, rowsum=rs, P=q["P"], beta=q["beta"], y=q["y"]))
                self.gemv_bytes += q["P"].numel() + M * q["K"] + 2 * M * q["N"] + 8 * M
            self.gemv_batches.append((B.make_quantized_batch(items), items))
        self.gemv_token = B.make_quantized_batch([it for _, items in self.gemv_batches
                                                  for it in items])
        self.launches = {"layer_batch": 2 * layers, "per_call": 2 * len(self.problems),
                         "token_batch": 2, "gemv_only": layers, "gemv_token": 1}
        self.graphs = {}

    def run(self, mode):
        B, eps, M = self.B, self.WL.RMS_EPS, self.M
        if mode == "layer_batch":
            for arr, ws, _ in self.layer_batches:
                B.bitlinear_forward_batch(arr, M, eps, workspace=ws)
        elif mode == "token_batch":
            B.bitlinear_forward_batch(self.token_batch, M, eps, workspace=self.token_ws)
        elif mode == "token_batch2":  # the same step on the second buffer set
            B.bitlinear_forward_batch(self.token_batch2, M, eps, workspace=self.token_ws)
        elif mode == "per_call":
            for q in self.problems:
                B.bitlinear_forward(q["x"], q["P"], q["beta"], gain=q["gain"], eps=eps, out=q["y"],
                                    workspace=q["ws"])
        elif mode == "gemv_only":
            for arr, _ in self.gemv_batches:
                B.bitlinear_forward_quantized_batch(arr, M)
        elif mode == "gemv_token":
            B.bitlinear_forward_quantized_batch(self.gemv_token, M)
        else:
            raise ValueError(mode)

    def capture(self, mode):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run(mode)  # eager once on the side stream (caches, attributes)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run(mode)
        torch.cuda.synchronize()
        self.graphs[mode] = g
        return g


class PrefillWorkload:
    """Config-4 prefill: M=4096 tokens through gate, up, down, q, o (RMSNorm,
    bf16 out).  Times the tensor-core GEMM launch on already-quantised codes and
    the whole forward (quantise + GEMM)."""

    def __init__(self, M=4096):
        import ternary_weight_bitlinear_b200 as B
        from ternary_weight_bitlinear_b200 import workloads as WL
        self.B, self.WL, self.M = B, WL, M
        self.items = []
        for name in WL.CONFIG4_PROJECTIONS:
            p = WL.PROJECTIONS[WL.PROJ_INDEX[name]]
            W = torch.from_numpy(WL.master_weights(p.N, p.K, WL.master_seed(0, name))).cuda()
            P, beta = B.bitlinear_pack(W)
            del W
            c = WL.config4_projection(name, M)
            x = torch.from_numpy(c["x"].view(np.int16)).view(torch.bfloat16).cuda()
            g = torch.from_numpy(c["gain"].view(np.int16)).view(torch.bfloat16).cuda()
            q, sx, rs = B.bitlinear_act_quant(x, g, WL.RMS_EPS)
            y = torch.empty((M, p.N), dtype=torch.bfloat16, device="cuda")
            ws = torch.empty(B.bitlinear_forward_workspace_size(M, p.K, p.N), dtype=torch.uint8,
                             device="cuda")
            self.items.append(dict(name=name, K=p.K, N=p.N, P=P, beta=float(beta.item()), x=x,
                                   g=g, q=q, sx=sx, rs=rs, y=y, ws=ws))

    def gemm(self, it):
        self.B.bitlinear_forward_quantized(it["q"], it["sx"], it["rs"], it["P"], it["beta"],
                                           out=it["y"])

    def forward(self, it):
        self.B.bitlinear_forward(it["x"], it["P"], it["beta"], gain=it["g"], eps=self.WL.RMS_EPS,
                                 out=it["y"], workspace=it["ws"])

    def measure(self, reps, warmup, world):
        peak, src = measured_int8_peak()
        out = {"workload": "prefill M=4096: gate/up 2560->6912, down 6912->2560, q/o "
                           "2560->2560; RMSNorm, bf16 out",
               "int8_peak_tops": peak, "peak_source": src, "projections": {}}
        tot_ops = tot_gemm_ms = tot_fwd_ms = 0.0
        for it in self.items:
            ops = 2.0 * self.M * it["N"] * it["K"]
            ms_g = timed(lambda: self.gemm(it), reps, warmup, world) / reps
            ms_f = timed(lambda: self.forward(it), reps, warmup, world) / reps
            out["projections"][it["name"]] = {
                "gemm_ms": ms_g, "gemm_tops": ops / ms_g / 1e9, "forward_ms": ms_f,
                "frac_of_int8_peak": ops / ms_g / 1e9 / peak}
            tot_ops += ops
            tot_gemm_ms += ms_g
            tot_fwd_ms += ms_f
        out["gemm_tops"] = tot_ops / tot_gemm_ms / 1e9
        out["frac_of_int8_peak"] = out["gemm_tops"] / peak
        out["tokens_per_s"] = self.M / (tot_fwd_ms / 1000.0)  # one pass over the 5 projections
        return out


class SkinnyWorkload:
    """Batched decode (5..64 tokens): every projection of all decoder layers
    with its own M-token input (per-token scales drawn from U(0.1, 10), no
    RMSNorm, bf16 out), over the packed weights of a DecodeWorkload.  Times the
    weight-streaming GEMV on already-quantised codes (its HBM roofline) and the
    whole batched forward (quantise + GEMV)."""

    def __init__(self, dec, M):
        import ternary_weight_bitlinear_b200 as B
        WL = dec.WL
        self.B, self.M = B, M
        items, qitems = [], []
        self.gemv_bytes = 0
        for q in dec.problems:
            c = WL.config3_projection(q["layer"], q["name"], M)
            x = torch.from_numpy(c["x"].view(np.int16)).view(torch.bfloat16).cuda()
            y = torch.empty((M, q["N"]), dtype=torch.bfloat16, device="cuda")
            items.append(dict(x=x, P=q["P"], beta=q["beta"], y=y))
            qq, sx, rs = B.bitlinear_act_quant(x)
            qitems.append(dict(q=qq, s_x=sx, rowsum=rs, P=q["P"], beta=q["beta"], y=y))
            self.gemv_bytes += q["P"].numel() + M * q["K"] + 2 * M * q["N"] + 8 * M
        self.items, self.qitems = items, qitems
        self.batch = B.make_batch(items)
        self.qbatch = B.make_quantized_batch(qitems)
        self.ws = torch.empty(B.bitlinear_forward_batch_workspace_size(self.batch, M),
                              dtype=torch.uint8, device="cuda")
        self.qws = torch.empty(max(16, B.bitlinear_quantized_batch_workspace_size(M)),
                               dtype=torch.uint8, device="cuda")
        self.graphs = {}
        for mode in ("gemv", "forward"):
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                self.run(mode)
            torch.cuda.current_stream().wait_stream(s)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.run(mode)
            torch.cuda.synchronize()
            self.graphs[mode] = g

    def run(self, mode):
        if mode == "gemv":
            self.B.bitlinear_forward_quantized_batch(self.qbatch, self.M, workspace=self.qws)
        else:
            self.B.bitlinear_forward_batch(self.batch, self.M, 0.0, workspace=self.ws)

    def measure(self, reps, warmup, world, hbm):
        ms_g = timed(self.graphs["gemv"].replay, reps, warmup, world) / reps
        ms_f = timed(self.graphs["forward"].replay, reps, warmup, world) / reps
        gbs = self.gemv_bytes / (ms_g / 1000.0) / 1e9
        return {"M": self.M, "gemv_us": ms_g * 1000.0, "gemv_gbs": gbs, "frac_of_hbm": gbs / hbm,
                "forward_us": ms_f * 1000.0, "tokens_per_s": world * self.M / (ms_f / 1000.0),
                "launches_per_step": {"gemv": (len(self.items) + 63) // 64,
                                      "forward": 1 + (len(self.items) + 63) // 64}}


class FfnChainWorkload:
    """Config 5: M=16 tokens through the FFN blocks of all 30 layers in order
    (RMSNorm -> gate, up -> relu(gate)^2 * up -> sub-norm -> down -> + residual),
    the packed gate/up/down weights of the headline workload.  Each layer is
    act_quant, one batched gate|up GEMV, relu2_mul, act_quant and the down
    GEMV with the residual epilogue: 5 launches per layer, captured in one
    graph that also restores the input."""

    def __init__(self, dec, M=16):
        import ternary_weight_bitlinear_b200 as B
        WL = dec.WL
        self.B, self.WL, self.M = B, WL, M
        byname = {(q["layer"], q["name"]): q for q in dec.problems}
        self.x0 = torch.from_numpy(WL.config5_input(M).view(np.int16)).view(torch.bfloat16).cuda()
        self.x = self.x0.clone()
        H, I = WL.HIDDEN, WL.INTERMEDIATE
        self.layers = []
        self.weight_bytes = 0
        for l in range(dec.layers):
            g, u, d = byname[(l, "gate")], byname[(l, "up")], byname[(l, "down")]
            gi = torch.from_numpy(WL.gain(H, 1000 * (l + 1) + 10).view(np.int16)).view(torch.bfloat16).cuda()
            gs = torch.from_numpy(WL.gain(I, 1000 * (l + 1) + 11).view(np.int16)).view(torch.bfloat16).cuda()
            self.layers.append(dict(g=g, u=u, d=d, gi=gi, gs=gs))
            self.weight_bytes += g["P"].numel() + u["P"].numel() + d["P"].numel()
        dev = "cuda"
        self.q1 = torch.empty((M, H), dtype=torch.int8, device=dev)
        self.s1 = torch.empty(M, dtype=torch.float32, device=dev)
        self.r1 = torch.empty(M, dtype=torch.int32, device=dev)
        self.a = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
        self.b = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
        self.z = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
        self.q2 = torch.empty((M, I), dtype=torch.int8, device=dev)
        self.s2 = torch.empty(M, dtype=torch.float32, device=dev)
        self.r2 = torch.empty(M, dtype=torch.int32, device=dev)
        self.ws = torch.empty(max(16, B.bitlinear_quantized_batch_workspace_size(M)),
                              dtype=torch.uint8, device=dev)
        for L in self.layers:
            L["gu"] = B.make_quantized_batch([
                dict(q=self.q1, s_x=self.s1, rowsum=self.r1, P=L["g"]["P"], beta=L["g"]["beta"], y=self.a),
                dict(q=self.q1, s_x=self.s1, rowsum=self.r1, P=L["u"]["P"], beta=L["u"]["beta"], y=self.b)])
            L["dn"] = B.make_quantized_batch([
                dict(q=self.q2, s_x=self.s2, rowsum=self.r2, P=L["d"]["P"], beta=L["d"]["beta"],
                     y=self.x, residual=self.x)])
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.run()
        torch.cuda.synchronize()

    def run(self):
        B, eps, M = self.B, self.WL.RMS_EPS, self.M
        self.x.copy_(self.x0)
        for L in self.layers:
            B.bitlinear_act_quant(self.x, L["gi"], eps, q=self.q1, s_x=self.s1, rowsum=self.r1)
            B.bitlinear_forward_quantized_batch(L["gu"], M, workspace=self.ws)
            B.bitlinear_relu2_mul(self.a, self.b, out=self.z)
            B.bitlinear_act_quant(self.z, L["gs"], eps, q=self.q2, s_x=self.s2, rowsum=self.r2)
            B.bitlinear_forward_quantized_batch(L["dn"], M, workspace=self.ws)

    def measure(self, reps, warmup, world, hbm):
        ms = timed(self.graph.replay, reps, warmup, world) / reps
        gbs = self.weight_bytes / (ms / 1000.0) / 1e9
        return {"workload": "config 5: M=%d tokens through the FFN blocks of %d BitNet-2B4T "
                            "layers in order (RMSNorm, gate|up, relu2*, sub-norm, down, "
                            "+residual); attention omitted" % (self.M, len(self.layers)),
                "chain_us": ms * 1000.0, "tokens_per_s": job_throughput(self.M, world, ms),
                "packed_weight_gbs": gbs, "frac_of_hbm": gbs / hbm,
                "launches_per_step": 5 * len(self.layers)}


def measured_int8_peak():
    """Dense int8 tensor peak: the measured bf16 GEMM burst x the nominal 2x ratio."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return 2.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 burst x 2 (nominal int8:bf16)"
    except Exception:
        return 2.0 * 1590.0, "fallback bf16 1.59 PF x 2"


def timed(fn, steps, warmup, world):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        fn()
    end.record()
    end.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end)  # ms


def timed_e2e(wl, steps, warmup, world):
    """Device time of `steps` end-to-end steps (host inputs in, host outputs out),
    pipelined over two buffer sets; ms, CUDA events on the compute stream."""
    graphs = (wl.graphs["token_batch"], wl.capture("token_batch2"))
    xs, ys = (wl.x_dev, wl.x_dev2), (wl.y_dev, wl.y_dev2)
    cmp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: [torch.cuda.Event() for _ in range(2)]
    x_in, done, y_out = ev(), ev(), ev()
    used = [False, False]

    def step(k):
        i = k % 2
        with torch.cuda.stream(h2d):
            if used[i]:
                h2d.wait_event(done[i])  # step k-2 has read this input buffer
            xs[i].copy_(wl.x_host, non_blocking=True)
            x_in[i].record(h2d)
        cmp.wait_event(x_in[i])
        if used[i]:
            cmp.wait_event(y_out[i])  # step k-2's outputs have left this buffer
        graphs[i].replay()
        done[i].record(cmp)
        with torch.cuda.stream(d2h):
            d2h.wait_event(done[i])
            wl.y_host.copy_(ys[i], non_blocking=True)
            y_out[i].record(d2h)
        used[i] = True

    for k in range(warmup):
        step(k)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(cmp)
    h2d.wait_stream(cmp)
    d2h.wait_stream(cmp)
    for k in range(steps):
        step(k)
    cmp.wait_stream(d2h)
    end.record(cmp)
    end.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    # the host outputs are the step's results
    assert torch.equal(wl.y_host, wl.y_dev.cpu()), "end-to-end outputs differ from the device run"
    return start.elapsed_time(end)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_sources_hash():
    h = hashlib.sha256()
    for name in DECODE_KERNEL_SOURCES:
        with open(os.path.join(ROOT, "ternary_weight_bitlinear_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(launches):
    """Per-launch DRAM traffic from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "decode_gemv_2b4t_m1.md")
    try:
        fields = {}
        with open(path) as f:
            for line in f:
                if ":" in line and line.startswith("- "):
                    k, v = line[2:].split(":", 1)
                    fields[k.strip()] = v.strip().strip("`")
        if fields.get("kernel_sources_sha256_16") != kernel_sources_hash():
            return None
        return float(fields["dram_bytes_per_step"]) / launches
    except Exception:
        return None


# ---------------------------------------------------------------------------
# CPU oracle baseline (rank 0, N=1 only)
# ---------------------------------------------------------------------------
def oracle_layer0_problems(WL, M=1):
    import oracle as O
    probs = []
    for p in WL.PROJECTIONS:
        Pm, beta = O.pack_master(WL.master_weights(p.N, p.K, WL.master_seed(0, p.name)))
        c = WL.config2_projection(0, p.name, M)
        probs.append((c, Pm, beta, p))
    return probs


def oracle_run(O, WL, probs, budget_s=None, per_step=None):
    """Time O.forward over the problems; return (seconds, tokens) where tokens is
    the fraction of one token's 30-layer work the timed calls covered."""
    units_token = token_work_units(WL, WL.LAYERS)
    t_total = 0.0
    units = 0
    i = 0
    while True:
        c, Pm, beta, p = probs[i % len(probs)]
        t0 = time.perf_counter()
        O.forward(c["x"], Pm, beta, gain=c["gain"], eps=WL.RMS_EPS, norm=True)
        t_total += time.perf_counter() - t0
        units += p.N * p.K
        i += 1
        if per_step is not None and i >= per_step:
            break
        if budget_s is not None and t_total >= budget_s and i >= len(probs):
            break
    return t_total, units / units_token


def cpu_baseline(budget_s):
    import oracle as O
    from ternary_weight_bitlinear_b200 import workloads as WL
    probs = oracle_layer0_problems(WL)
    secs, tokens = oracle_run(O, WL, probs, budget_s=budget_s)
    return {"value": tokens / secs, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": "layer 0's seven M=1 BitLinear forwards (same shapes, seeds and "
                      "RMSNorm as the GPU workload), repeated for %.1f s on one host core; "
                      "tokens = covered MACs / one token's 30-layer MACs" % secs}


def reference_arm(args, world, rank):
    """The oracle as the reference arm: same workload, metric and unit."""
    if rank != 0:
        return
    import oracle as O
    from ternary_weight_bitlinear_b200 import workloads as WL
    probs = oracle_layer0_problems(WL)
    # each step: a bounded sample (7 forwards for short runs, 1 for long ones)
    per_step = 7 if args.steps <= 60 else 1
    for _ in range(args.warmup):
        oracle_run(O, WL, probs, per_step=per_step)
    secs = 0.0
    tokens = 0.0
    for s in range(args.steps):
        rot = probs[(s * per_step) % 7:] + probs[:(s * per_step) % 7]
        t, tk = oracle_run(O, WL, rot, per_step=per_step)
        secs += t
        tokens += tk
    value = tokens / secs
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * secs / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": workload_config(args, None),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": "%d oracle BitLinear forward(s) per step from layer 0's "
                                       "seven projections, rotating" % per_step},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(args, wl):
    cfg = {"workload": "decode M=1: one token through the 7 BitLinear projections "
                       "(q,k,v,o 2560->2560/640, gate/up 2560->6912, down 6912->2560) of each "
                       "of the 30 BitNet-2B4T layers (independent inputs per projection); "
                       "RMSNorm, int8 absmax, ternary matmul, bf16 out; all 210 forwards in "
                       "one batched call (2 launches: quantise, GEMV)",
           "M": 1, "layers": args.layers, "hidden": 2560, "intermediate": 6912,
           "parallelism": "replicas" if args.gpus > 1 else "single",
           "l2": "no flush: the 521 MB of packed weights per step exceed the 126 MB L2"}
    if wl is not None:
        cfg["packed_weight_bytes_per_step"] = wl.weight_bytes
        cfg["algorithmic_bytes_per_step"] = wl.step_bytes
    return cfg


# ---------------------------------------------------------------------------
def main():
    args = parse_args()
    world, rank, local = dist_setup()
    if args.impl == "reference":
        reference_arm(args, world, rank)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    from __graft_entry__ import build
    if rank == 0:
        build()
    barrier(world)
    wl = DecodeWorkload(args.layers)
    # capture order fixes the launch order that profiles/ commands count on
    for mode in ("layer_batch", "gemv_only", "per_call", "token_batch", "gemv_token"):
        wl.capture(mode)
    head = wl.graphs["token_batch"]

    # device-resident timing of the headline: all 210 projections of the token
    # in one batched forward call (one quantise launch + one GEMV launch)
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms = timed(head.replay, args.steps, args.warmup, world)
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    value = job_throughput(wl.M * args.steps, world, ms)

    # the GEMV kernel alone on the same batch (pre-quantised codes): its roofline
    ms_gemv = max_over_ranks(timed(wl.graphs["gemv_token"].replay, args.steps, args.warmup, world),
                             world)
    variants = {}
    for mode in ("layer_batch", "per_call", "gemv_only"):
        t = max_over_ranks(timed(wl.graphs[mode].replay, args.steps, args.warmup, world), world)
        variants[mode] = {"tokens_per_s": job_throughput(wl.M * args.steps, world, t),
                          "ms_per_step": t / args.steps, "launches_per_step": wl.launches[mode]}
    variants["gemv_only"]["note"] = ("the layer_batch GEMV launches alone (17.4 MB each): "
                                     "bound by per-launch ramp, see profiles/")

    # end to end: every step copies its inputs from pinned host memory, runs the
    # forwards and copies its outputs back to pinned host memory.  Steps
    # alternate between two buffer sets, with the copies on their own streams,
    # so step k+1's input copy and step k-1's output copy overlap step k.
    ms_e2e = max_over_ranks(timed_e2e(wl, args.steps, args.warmup, world), world)
    e2e_value = job_throughput(wl.M * args.steps, world, ms_e2e)

    hbm, hbm_src = measured_peaks()
    skinny = None
    if not args.no_skinny:
        skinny = {"workload": "batched decode: M tokens through the 210 projections of 30 "
                              "BitNet-2B4T layers (independent inputs, per-token scales "
                              "U(0.1, 10)), no RMSNorm, bf16 out; weights of the headline",
                  "by_M": {}}
        for Ms in (8, 32, 64):
            sw = SkinnyWorkload(wl, Ms)
            skinny["by_M"][str(Ms)] = sw.measure(max(3, min(args.steps, 20)), max(args.warmup, 2),
                                                 world, hbm)
            del sw
    ffn = None
    if not args.no_skinny:
        fw = FfnChainWorkload(wl)
        ffn = fw.measure(max(3, min(args.steps, 20)), max(args.warmup, 2), world, hbm)
        del fw
    prefill = None
    if not args.no_prefill:
        pw = PrefillWorkload()
        prefill = pw.measure(max(3, min(args.steps, 20)), max(args.warmup, 2), world)

    status = wl.B.bitlinear_device_status()
    if status != 0:
        raise RuntimeError("device status %d after the timed region" % status)

    gemv_launch_ms = ms_gemv / args.steps
    bytes_per_launch = wl.gemv_bytes
    achieved = bytes_per_launch / (gemv_launch_ms / 1000.0) / 1e9
    traffic = recorded_traffic(1)
    variants["token_batch_step_gbs"] = wl.step_bytes / (ms_step / 1000.0) / 1e9

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "int8", "data": "synthetic", "config": workload_config(args, wl),
                "roofline": {"bound": "hbm",
                             "kernel": "decode_batch_kernel (the token's 210 projections in one launch)",
                             "achieved": achieved, "peak": hbm, "peak_source": hbm_src,
                             "unit": "GB/s", "frac": achieved / hbm, "traffic": traffic,
                             "launch_us": gemv_launch_ms * 1000.0,
                             "bytes_per_launch": bytes_per_launch},
                "variants": variants,
                "skinny": skinny,
                "ffn_chain": ffn,
                "prefill": prefill,
                "e2e": {"value": e2e_value, "unit": "tokens/s",
                        "h2d_bytes_per_step": wl.h2d_bytes, "d2h_bytes_per_step": wl.d2h_bytes,
                        "note": "pinned host x in and y out every step, through the public "
                                "batched forward; two buffer sets, copies on their own "
                                "streams overlap the neighbouring steps' compute"},
                "gpu_launches": wl.launches["token_batch"] * args.steps,
                "clocks": clk.result()}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        wl.graphs.clear()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
