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
import math
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
NOMINAL_HBM_GBS = 8000.0      # B200 HBM3e, public figure
NOMINAL_INT8_TOPS = 4500.0    # B200 dense int8 tensor, public figure
HEADLINE_MIN_S = 0.5          # device time the headline's timed region covers at least
LEG_REPS = 100                # repeats of every other timed leg


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
    ap.add_argument("--no-comparator", action="store_true",
                    help="skip the bf16 dequantised-matmul comparator")
    ap.add_argument("--passes", type=int, default=0,
                    help="token passes per headline step (0: enough for %.1f s of device time)"
                    % HEADLINE_MIN_S)
    ap.add_argument("--reps", type=int, default=LEG_REPS,
                    help="timed repeats of every other leg (profiling runs use a few)")
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

    def gate_up_pair(self, l):
        """Layer l's gate and up projections packed as one pair (cached)."""
        if not hasattr(self, "_pairs"):
            self._pairs = {}
        if l not in self._pairs:
            WL = self.WL
            p = WL.PROJECTIONS[WL.PROJ_INDEX["gate"]]
            Wg = torch.from_numpy(WL.master_weights(p.N, p.K, WL.master_seed(l, "gate"))).cuda()
            Wu = torch.from_numpy(WL.master_weights(p.N, p.K, WL.master_seed(l, "up"))).cuda()
            P2, b2 = self.B.bitlinear_pack_gate_up(Wg, Wu)
            del Wg, Wu
            self._pairs[l] = (P2, [float(v) for v in b2.cpu()])
        return self._pairs[l]

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
                "frac_of_int8_peak": ops / ms_g / 1e9 / peak,
                "frac_of_nominal_int8": ops / ms_g / 1e9 / NOMINAL_INT8_TOPS}
            tot_ops += ops
            tot_gemm_ms += ms_g
            tot_fwd_ms += ms_f
        out["gemm_tops"] = tot_ops / tot_gemm_ms / 1e9
        out["frac_of_int8_peak"] = out["gemm_tops"] / peak
        out["frac_of_nominal_int8"] = out["gemm_tops"] / NOMINAL_INT8_TOPS
        out["reps"] = reps
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
                "frac_of_nominal_hbm": gbs / NOMINAL_HBM_GBS, "reps": reps,
                "forward_us": ms_f * 1000.0, "tokens_per_s": world * self.M / (ms_f / 1000.0),
                "launches_per_step": {"gemv": (len(self.items) + 63) // 64,
                                      "forward": 1 + (len(self.items) + 63) // 64}}


class FfnChainWorkload:
    """Config 5: M=16 tokens through the FFN blocks of all 30 layers in order
    (RMSNorm -> gate|up -> relu(gate)^2 * up -> sub-norm -> down -> + residual).
    Each layer is act_quant, the fused gate|up pass (one read of the pair's
    packed weights, relu^2*up in the epilogue), act_quant and the down
    projection with the residual epilogue: 4 launches per layer, captured in
    one graph that also restores the input."""

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
            P2, b2 = dec.gate_up_pair(l)
            d = byname[(l, "down")]
            gi = torch.from_numpy(WL.gain(H, 1000 * (l + 1) + 10).view(np.int16)).view(torch.bfloat16).cuda()
            gs = torch.from_numpy(WL.gain(I, 1000 * (l + 1) + 11).view(np.int16)).view(torch.bfloat16).cuda()
            self.layers.append(dict(P2=P2, bg=b2[0], bu=b2[1], d=d, gi=gi, gs=gs))
            self.weight_bytes += P2.numel() + d["P"].numel()
        dev = "cuda"
        self.q1 = torch.empty((M, H), dtype=torch.int8, device=dev)
        self.s1 = torch.empty(M, dtype=torch.float32, device=dev)
        self.r1 = torch.empty(M, dtype=torch.int32, device=dev)
        self.z = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
        self.q2 = torch.empty((M, I), dtype=torch.int8, device=dev)
        self.s2 = torch.empty(M, dtype=torch.float32, device=dev)
        self.r2 = torch.empty(M, dtype=torch.int32, device=dev)
        self.ws = torch.empty(max(16, B.bitlinear_quantized_batch_workspace_size(M)),
                              dtype=torch.uint8, device=dev)
        for L in self.layers:
            L["dn"] = B.make_quantized_batch([
                dict(q=self.q2, s_x=self.s2, rowsum=self.r2, P=L["d"]["P"], beta=L["d"]["beta"],
                     y=self.x, residual=self.x)])
        self.graph = capture_graph(self.run)

    def unfused(self, dec):
        """The same chain with gate and up as two problems of one batched
        call, then relu2_mul: 5 launches a layer (the control of the fused pass)."""
        B = self.B
        byname = {(q["layer"], q["name"]): q for q in dec.problems}
        M, I = self.M, self.WL.INTERMEDIATE
        self.a = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
        self.b = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
        for l, L in enumerate(self.layers):
            g, u = byname[(l, "gate")], byname[(l, "up")]
            L["gu"] = B.make_quantized_batch([
                dict(q=self.q1, s_x=self.s1, rowsum=self.r1, P=g["P"], beta=g["beta"], y=self.a),
                dict(q=self.q1, s_x=self.s1, rowsum=self.r1, P=u["P"], beta=u["beta"], y=self.b)])
        self.graph_unfused = capture_graph(self.run_unfused)

    def run_unfused(self):
        B, eps, M = self.B, self.WL.RMS_EPS, self.M
        self.x.copy_(self.x0)
        for L in self.layers:
            B.bitlinear_act_quant(self.x, L["gi"], eps, q=self.q1, s_x=self.s1, rowsum=self.r1)
            B.bitlinear_forward_quantized_batch(L["gu"], M, workspace=self.ws)
            B.bitlinear_relu2_mul(self.a, self.b, out=self.z)
            B.bitlinear_act_quant(self.z, L["gs"], eps, q=self.q2, s_x=self.s2, rowsum=self.r2)
            B.bitlinear_forward_quantized_batch(L["dn"], M, workspace=self.ws)

    def measure_unfused(self, reps, warmup, world):
        ms = timed(self.graph_unfused.replay, reps, warmup, world) / reps
        return {"chain_us": ms * 1000.0, "tokens_per_s": job_throughput(self.M, world, ms),
                "launches_per_step": 5 * len(self.layers), "reps": reps}

    def run(self):
        B, eps, M = self.B, self.WL.RMS_EPS, self.M
        self.x.copy_(self.x0)
        for L in self.layers:
            B.bitlinear_act_quant(self.x, L["gi"], eps, q=self.q1, s_x=self.s1, rowsum=self.r1)
            B.bitlinear_forward_gate_up(self.q1, self.s1, self.r1, L["P2"], L["bg"], L["bu"],
                                        out=self.z, workspace=self.ws)
            B.bitlinear_act_quant(self.z, L["gs"], eps, q=self.q2, s_x=self.s2, rowsum=self.r2)
            B.bitlinear_forward_quantized_batch(L["dn"], M, workspace=self.ws)

    def measure(self, reps, warmup, world, hbm):
        ms = timed(self.graph.replay, reps, warmup, world) / reps
        gbs = self.weight_bytes / (ms / 1000.0) / 1e9
        return {"workload": "config 5: M=%d tokens through the FFN blocks of %d BitNet-2B4T "
                            "layers in order (RMSNorm, fused gate|up -> relu2*up, sub-norm, down, "
                            "+residual); attention omitted" % (self.M, len(self.layers)),
                "chain_us": ms * 1000.0, "tokens_per_s": job_throughput(self.M, world, ms),
                "packed_weight_gbs": gbs, "frac_of_hbm": gbs / hbm,
                "frac_of_nominal_hbm": gbs / NOMINAL_HBM_GBS, "reps": reps,
                "launches_per_step": 4 * len(self.layers)}


class DecodeChainWorkload:
    """One token (M=1) through the 30 decoder layers in order, every step
    waiting on the one before: per layer the RMS-normalised layer input is
    quantised once for the attention projections (q|k|v as one batched call,
    then o -- attention itself omitted, so o reads the same quantised input --
    whose output is added to the residual stream), then the FFN block
    (RMSNorm, fused gate|up -> relu^2*up, sub-norm, down + residual).  Seven
    launches per layer; every packed weight of the token streams once."""

    def __init__(self, dec):
        import ternary_weight_bitlinear_b200 as B
        WL = dec.WL
        self.B, self.WL = B, WL
        byname = {(q["layer"], q["name"]): q for q in dec.problems}
        H, I = WL.HIDDEN, WL.INTERMEDIATE
        dev = "cuda"
        self.x0 = torch.from_numpy(WL.activations(1, H, seed=7).view(np.int16)).view(torch.bfloat16).cuda()
        self.x = self.x0.clone()
        self.qa = torch.empty((1, H), dtype=torch.int8, device=dev)
        self.qf = torch.empty((1, H), dtype=torch.int8, device=dev)
        self.qs = torch.empty((1, I), dtype=torch.int8, device=dev)
        self.sv = torch.empty((3, 1), dtype=torch.float32, device=dev)
        self.rv = torch.empty((3, 1), dtype=torch.int32, device=dev)
        self.qkv = [torch.empty((1, byname[(0, n)]["N"]), dtype=torch.bfloat16, device=dev)
                    for n in ("q", "k", "v")]
        self.z = torch.empty((1, I), dtype=torch.bfloat16, device=dev)
        self.layers = []
        self.weight_bytes = 0
        for l in range(dec.layers):
            P2, b2 = dec.gate_up_pair(l)
            g = lambda K, seed: torch.from_numpy(WL.gain(K, seed).view(np.int16)).view(torch.bfloat16).cuda()
            L = dict(ga=g(H, 1000 * (l + 1) + 12), gf=g(H, 1000 * (l + 1) + 10),
                     gs=g(I, 1000 * (l + 1) + 11), P2=P2, bg=b2[0], bu=b2[1])
            L["qkv"] = B.make_quantized_batch([
                dict(q=self.qa, s_x=self.sv[0], rowsum=self.rv[0], P=byname[(l, n)]["P"],
                     beta=byname[(l, n)]["beta"], y=y) for n, y in zip(("q", "k", "v"), self.qkv)])
            L["o"] = B.make_quantized_batch([
                dict(q=self.qa, s_x=self.sv[0], rowsum=self.rv[0], P=byname[(l, "o")]["P"],
                     beta=byname[(l, "o")]["beta"], y=self.x, residual=self.x)])
            L["down"] = B.make_quantized_batch([
                dict(q=self.qs, s_x=self.sv[2], rowsum=self.rv[2], P=byname[(l, "down")]["P"],
                     beta=byname[(l, "down")]["beta"], y=self.x, residual=self.x)])
            self.layers.append(L)
            self.weight_bytes += sum(byname[(l, n)]["P"].numel() for n in ("q", "k", "v", "o", "down"))
            self.weight_bytes += P2.numel()
        self.graph = capture_graph(self.run)

    def run(self):
        B, eps = self.B, self.WL.RMS_EPS
        self.x.copy_(self.x0)
        for L in self.layers:
            B.bitlinear_act_quant(self.x, L["ga"], eps, q=self.qa, s_x=self.sv[0], rowsum=self.rv[0])
            B.bitlinear_forward_quantized_batch(L["qkv"], 1)
            B.bitlinear_forward_quantized_batch(L["o"], 1)
            B.bitlinear_act_quant(self.x, L["gf"], eps, q=self.qf, s_x=self.sv[1], rowsum=self.rv[1])
            B.bitlinear_forward_gate_up(self.qf, self.sv[1], self.rv[1], L["P2"], L["bg"], L["bu"],
                                        out=self.z)
            B.bitlinear_act_quant(self.z, L["gs"], eps, q=self.qs, s_x=self.sv[2], rowsum=self.rv[2])
            B.bitlinear_forward_quantized_batch(L["down"], 1)

    def with_attention(self, dec, L=1024):
        """The full dependent decode step of the 2B4T decoder layer: per layer
        the input norm + q|k|v (k and v written straight into row L - 1 of the
        layer's key/value cache), RoPE of q and of that key row, grouped-query
        attention over the L cached positions, attn_sub_norm + o + residual,
        then the FFN block as above.  Twelve launches a layer; the caches hold
        seeded random keys and values for the L - 1 earlier positions."""
        B, WL = self.B, self.WL
        byname = {(q["layer"], q["name"]): q for q in dec.problems}
        H, Hq, Hkv, d = WL.HIDDEN, WL.Q_HEADS, WL.KV_HEADS, WL.HEAD_DIM
        dev = "cuda"
        self.L_att = L
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
        self.qbuf = torch.empty((1, H), dtype=torch.bfloat16, device=dev)
        self.att = torch.empty(H, dtype=torch.bfloat16, device=dev)
        self.qo = torch.empty((1, H), dtype=torch.int8, device=dev)
        self.svo = torch.empty(1, dtype=torch.float32, device=dev)
        self.rvo = torch.empty(1, dtype=torch.int32, device=dev)
        self.pos = torch.full((1,), L - 1, dtype=torch.int32, device=dev)
        self.att_ws = torch.empty(max(16, B.bitlinear_attn_decode_workspace_size(L, Hq, Hkv, d)),
                                  dtype=torch.uint8, device=dev)
        self.kv_bytes = 0
        for l, Lr in enumerate(self.layers):
            _, k0, v0 = WL.attention_decode_inputs(L, seed=5000 + 10 * l)
            Lr["kc"], Lr["vc"] = bf(k0), bf(v0)
            krow, vrow = Lr["kc"][L - 1].reshape(1, Hkv * d), Lr["vc"][L - 1].reshape(1, Hkv * d)
            Lr["krow"] = krow
            Lr["gsub"] = torch.from_numpy(WL.gain(H, 1000 * (l + 1) + 13).view(np.int16)).view(
                torch.bfloat16).cuda()
            Lr["qkv_att"] = B.make_quantized_batch([
                dict(q=self.qa, s_x=self.sv[0], rowsum=self.rv[0], P=byname[(l, n)]["P"],
                     beta=byname[(l, n)]["beta"], y=y)
                for n, y in zip(("q", "k", "v"), (self.qbuf, krow, vrow))])
            Lr["o_att"] = B.make_quantized_batch([
                dict(q=self.qo, s_x=self.svo, rowsum=self.rvo, P=byname[(l, "o")]["P"],
                     beta=byname[(l, "o")]["beta"], y=self.x, residual=self.x)])
            self.kv_bytes += L * Hkv * d * 2 * 2
        self.att_scale = 1.0 / math.sqrt(d)
        self.agraph = capture_graph(self.run_attention)

    def run_attention(self):
        B, WL, eps = self.B, self.WL, self.WL.RMS_EPS
        self.x.copy_(self.x0)
        for Lr in self.layers:
            B.bitlinear_act_quant(self.x, Lr["ga"], eps, q=self.qa, s_x=self.sv[0], rowsum=self.rv[0])
            B.bitlinear_forward_quantized_batch(Lr["qkv_att"], 1)
            B.bitlinear_rope(self.qbuf, self.pos, WL.Q_HEADS, 500000.0, out=self.qbuf)
            B.bitlinear_rope(Lr["krow"], self.pos, WL.KV_HEADS, 500000.0, out=Lr["krow"])
            B.bitlinear_attn_decode(self.qbuf.reshape(-1), Lr["kc"], Lr["vc"], self.L_att, WL.Q_HEADS,
                                    WL.KV_HEADS, self.att_scale, out=self.att, workspace=self.att_ws)
            B.bitlinear_act_quant(self.att.reshape(1, -1), Lr["gsub"], eps, q=self.qo, s_x=self.svo,
                                  rowsum=self.rvo)
            B.bitlinear_forward_quantized_batch(Lr["o_att"], 1)
            B.bitlinear_act_quant(self.x, Lr["gf"], eps, q=self.qf, s_x=self.sv[1], rowsum=self.rv[1])
            B.bitlinear_forward_gate_up(self.qf, self.sv[1], self.rv[1], Lr["P2"], Lr["bg"], Lr["bu"],
                                        out=self.z)
            B.bitlinear_act_quant(self.z, Lr["gs"], eps, q=self.qs, s_x=self.sv[2], rowsum=self.rv[2])
            B.bitlinear_forward_quantized_batch(Lr["down"], 1)

    def measure_attention(self, reps, warmup, world, hbm):
        ms = timed(self.agraph.replay, reps, warmup, world) / reps
        tot = self.weight_bytes + self.kv_bytes
        gbs = tot / (ms / 1000.0) / 1e9
        return {"workload": "full dependent decode step: one token through the %d BitNet-2B4T "
                            "layers in order, each norm + q|k|v, RoPE, GQA attention over a "
                            "%d-position cache, attn_sub_norm + o + residual, then the FFN block"
                            % (len(self.layers), self.L_att),
                "token_us": ms * 1000.0, "tokens_per_s": job_throughput(1, world, ms),
                "bytes": tot, "gbs": gbs, "frac_of_hbm": gbs / hbm, "reps": reps,
                "launches_per_step": 12 * len(self.layers)}

    def persistent(self, dec):
        """The same token's steps as one persistent launch (3 steps a layer:
        q|k|v + o, gate|up, down), on a second pair of residual buffers."""
        B, WL = self.B, self.WL
        byname = {(q["layer"], q["name"]): q for q in dec.problems}
        H, I = WL.HIDDEN, WL.INTERMEDIATE
        self.pxa = self.x0.reshape(-1).clone()
        self.pxb = torch.empty_like(self.pxa)
        self.pz = torch.empty(I, dtype=torch.bfloat16, device="cuda")
        pqkv = [t.reshape(-1) for t in self.qkv]
        steps = []
        for l, L in enumerate(self.layers):
            steps.append(dict(x=self.pxa, gain=L["ga"], eps=WL.RMS_EPS, problems=[
                dict(P=byname[(l, n)]["P"], beta=byname[(l, n)]["beta"], y=y)
                for n, y in zip(("q", "k", "v"), pqkv)] + [
                dict(P=byname[(l, "o")]["P"], beta=byname[(l, "o")]["beta"], y=self.pxb,
                     residual=self.pxa)]))
            steps.append(dict(x=self.pxb, gain=L["gf"], eps=WL.RMS_EPS, problems=[
                dict(P=L["P2"], beta=L["bg"], beta_up=L["bu"], y=self.pz, kind="gate_up")]))
            steps.append(dict(x=self.pz, gain=L["gs"], eps=WL.RMS_EPS, problems=[
                dict(P=byname[(l, "down")]["P"], beta=byname[(l, "down")]["beta"], y=self.pxa,
                     residual=self.pxb)]))
        self.chain = B.make_chain(steps)
        self.chain_ws = B.bitlinear_decode_chain_prepare(self.chain)
        self.pgraph = capture_graph(self.run_persistent)

    def run_persistent(self):
        self.pxa.copy_(self.x0.reshape(-1))
        self.B.bitlinear_decode_chain_run(self.chain_ws, len(self.chain))

    def measure_persistent(self, reps, warmup, world, hbm):
        ms = timed(self.pgraph.replay, reps, warmup, world) / reps
        gbs = self.weight_bytes / (ms / 1000.0) / 1e9
        return {"workload": "dependent decode as one persistent launch: the token's %d steps "
                            "(per layer q|k|v + o, fused gate|up, down; each step quantises its "
                            "input in every CTA; grid barrier between steps); attention omitted"
                            % len(self.chain),
                "token_us": ms * 1000.0, "tokens_per_s": job_throughput(1, world, ms),
                "packed_weight_gbs": gbs, "frac_of_hbm": gbs / hbm,
                "frac_of_nominal_hbm": gbs / NOMINAL_HBM_GBS, "reps": reps,
                "launches_per_step": 1}

    def measure(self, reps, warmup, world, hbm):
        ms = timed(self.graph.replay, reps, warmup, world) / reps
        gbs = self.weight_bytes / (ms / 1000.0) / 1e9
        return {"workload": "dependent decode: one token through the %d BitNet-2B4T layers in "
                            "order (quantise, q|k|v, o + residual, quantise, fused gate|up, "
                            "quantise, down + residual per layer); attention omitted"
                            % len(self.layers),
                "token_us": ms * 1000.0, "tokens_per_s": job_throughput(1, world, ms),
                "packed_weight_gbs": gbs, "frac_of_hbm": gbs / hbm,
                "frac_of_nominal_hbm": gbs / NOMINAL_HBM_GBS, "reps": reps,
                "launches_per_step": 7 * len(self.layers),
                "packed_weight_bytes": self.weight_bytes}


class Bf16Comparator:
    """The offline-dequantised path the pages describe for the stock
    transformers integration, for context: packed weights unpacked to bf16
    once (t * beta), then a dense bf16 matmul (torch / cuBLAS) per projection,
    activations left in bf16.  Timed at the decode shapes (one token through
    the seven projections of one layer, repeated for 30 layers' worth of
    distinct weights) and at the prefill gate shape (M = 4096)."""

    def __init__(self, dec):
        import ternary_weight_bitlinear_b200 as B
        self.dec = dec
        self.w = []
        for q in dec.problems:  # all 210 projections: 4.2 GB of bf16 weights, > L2
            t = B.bitlinear_unpack(q["P"]).to(torch.bfloat16)
            self.w.append((t * torch.tensor(q["beta"], dtype=torch.bfloat16, device="cuda"), q))
        self.xs = [torch.randn((1, q["K"]), device="cuda", dtype=torch.bfloat16) for _, q in self.w]
        self.ys = [torch.empty((1, q["N"]), device="cuda", dtype=torch.bfloat16) for _, q in self.w]
        self.graph = capture_graph(self.run)
        gate = next(q for _, q in self.w if q["name"] == "gate")
        self.wg = next(w for w, q in self.w if q is gate)
        self.xp = torch.randn((4096, gate["K"]), device="cuda", dtype=torch.bfloat16)
        self.yp = torch.empty((4096, gate["N"]), device="cuda", dtype=torch.bfloat16)

    def run(self):
        for (w, _), x, y in zip(self.w, self.xs, self.ys):
            torch.matmul(x, w.t(), out=y)

    def measure(self, reps, warmup, world):
        ms = timed(self.graph.replay, reps, warmup, world) / reps
        wbytes = sum(w.numel() * 2 for w, _ in self.w)
        ms_p = timed(lambda: torch.matmul(self.xp, self.wg.t(), out=self.yp), reps, warmup,
                     world) / reps
        ops = 2.0 * 4096 * self.wg.shape[0] * self.wg.shape[1]
        return {"workload": "bf16 matmuls of the dequantised weights (torch / cuBLAS): one "
                            "token through all 210 projections; prefill M=4096 gate",
                "decode_token_us": ms * 1000.0, "decode_tokens_per_s": 1000.0 / ms,
                "decode_bf16_weight_gbs": wbytes / (ms / 1000.0) / 1e9,
                "prefill_gate_us": ms_p * 1000.0, "prefill_gate_tflops": ops / ms_p / 1e9,
                "reps": reps}


class AttentionWorkload:
    """The attention block of one decode token at the 2B4T head shapes (20
    query heads, 5 key/value heads of 128): RoPE of its q and k rows, then the
    grouped-query attention over an L-position key/value cache (the model's
    2048 positions at most), both through the public entry points, captured
    in a CUDA graph of `calls` token-layers.  Bytes per call: the L cached key
    and value rows read once (L * 640 * 2 * 2) plus q, k and the output."""

    def __init__(self, L, calls=30):
        import ternary_weight_bitlinear_b200 as B
        from ternary_weight_bitlinear_b200 import workloads as WL
        self.B, self.L, self.calls = B, L, calls
        H, Hkv, d = WL.Q_HEADS, WL.KV_HEADS, WL.HEAD_DIM
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
        q, k, v = WL.attention_decode_inputs(L, seed=L + 3)
        self.q, self.k, self.v = dev(q), dev(k), dev(v)
        self.knew = self.k[L - 1].reshape(1, Hkv * d)  # the token's own key row, rotated in place
        self.qm = self.q.reshape(1, H * d)
        self.pos = torch.full((1,), L - 1, dtype=torch.int32, device="cuda")
        self.out = torch.empty(H * d, dtype=torch.bfloat16, device="cuda")
        self.ws = torch.empty(max(16, B.bitlinear_attn_decode_workspace_size(L, H, Hkv, d)),
                              dtype=torch.uint8, device="cuda")
        self.scale = 1.0 / math.sqrt(d)
        self.H, self.Hkv = H, Hkv
        self.bytes = L * Hkv * d * 2 * 2 + 2 * H * d * 2 + Hkv * d * 2 * 2
        self.graph = capture_graph(self.run)

    def run(self):
        B = self.B
        for _ in range(self.calls):
            B.bitlinear_rope(self.qm, self.pos, self.H, 500000.0, out=self.qm)
            B.bitlinear_rope(self.knew, self.pos, self.Hkv, 500000.0, out=self.knew)
            B.bitlinear_attn_decode(self.q, self.k, self.v, self.L, self.H, self.Hkv, self.scale,
                                    out=self.out, workspace=self.ws)

    def measure(self, reps, warmup, world, hbm):
        ms = timed(self.graph.replay, reps, warmup, world) / reps / self.calls
        gbs = self.bytes / (ms / 1000.0) / 1e9
        return {"L": self.L, "layer_us": ms * 1000.0, "gbs": gbs, "frac_of_hbm": gbs / hbm,
                "launches_per_layer": 4, "reps": reps}


def capture_graph(fn):
    """Run fn once on a side stream (caches, attributes), then capture it."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


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
    """The oracle timed on the host cores: its OpenMP build on every core (the
    reported value) and the plain build on one core, half the budget each,
    plus one-off timings of config 1 and of a config-4 sample."""
    import oracle as O
    from ternary_weight_bitlinear_b200 import workloads as WL
    probs = oracle_layer0_problems(WL)
    cores = os.cpu_count() or 1
    O.set_parallel(True)
    secs_n, tokens_n = oracle_run(O, WL, probs, budget_s=budget_s / 2)
    # config 4 sample: 16 of the 4096 rows of the gate projection, all cores
    c4 = WL.config4_projection("gate")
    Pg, bg = O.pack_master(WL.master_weights(6912, 2560, WL.master_seed(0, "gate")))
    t0 = time.perf_counter()
    O.forward(c4["x"][:16], Pg, bg, gain=c4["gain"], eps=WL.RMS_EPS, norm=True)
    c4_row_s = (time.perf_counter() - t0) / 16
    O.set_parallel(False)
    secs_1, tokens_1 = oracle_run(O, WL, probs, budget_s=budget_s / 2)
    c1 = WL.config1()
    P1, b1 = O.pack_master(c1["W"])
    t0 = time.perf_counter()
    O.forward(c1["x"], P1, b1)
    c1_ms = (time.perf_counter() - t0) * 1000.0
    return {"value": tokens_n / secs_n, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "layer 0's seven M=1 BitLinear forwards (same shapes, seeds and RMSNorm "
                      "as the GPU workload), repeated for %.1f s with the oracle's OpenMP "
                      "build on %d host cores; tokens = covered MACs / one token's 30-layer "
                      "MACs" % (secs_n, cores),
            "value_1core": tokens_1 / secs_1,
            "config1_forward_ms_1core": c1_ms,
            "config4_gate_s_per_row_all_cores": c4_row_s,
            "config4_gate_projected_s_all_cores": c4_row_s * 4096}


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
            "passes_per_step": 1,
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
           "l2": "no flush: the 521 MB of packed weights per token pass exceed the 126 MB L2"}
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
    # in one batched forward call (one quantise launch + one GEMV launch).  A
    # step is `passes` back-to-back passes of that call, enough that the K
    # timed steps cover at least HEADLINE_MIN_S of device time.
    if args.passes > 0:
        passes = args.passes
    else:
        probe_ms = timed(head.replay, 20, max(args.warmup, 3), world) / 20
        passes = int(max(1, min(2000, np.ceil(HEADLINE_MIN_S * 1000.0 / (args.steps * probe_ms)))))
        passes = int(max_over_ranks(passes, world))

    def head_step():
        for _ in range(passes):
            head.replay()

    with ClockSampler(torch.cuda.current_device()) as clk:
        ms = timed(head_step, args.steps, args.warmup, world)
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    value = job_throughput(wl.M * passes * args.steps, world, ms)

    reps, rw = args.reps, max(args.warmup, 3)
    # the GEMV kernel alone on the same batch (pre-quantised codes): its roofline
    ms_gemv = max_over_ranks(timed(wl.graphs["gemv_token"].replay, reps, rw, world), world)
    variants = {}
    for mode in ("layer_batch", "per_call", "gemv_only"):
        t = max_over_ranks(timed(wl.graphs[mode].replay, reps, rw, world), world)
        variants[mode] = {"tokens_per_s": job_throughput(wl.M * reps, world, t),
                          "ms_per_pass": t / reps, "launches_per_pass": wl.launches[mode]}
    variants["gemv_only"]["note"] = ("the layer_batch GEMV launches alone (17.4 MB each): "
                                     "bound by per-launch ramp, see profiles/")

    # end to end: every pass copies its inputs from pinned host memory, runs the
    # forwards and copies its outputs back to pinned host memory.  Passes
    # alternate between two buffer sets, with the copies on their own streams,
    # so pass k+1's input copy and pass k-1's output copy overlap pass k.
    ms_e2e = max_over_ranks(timed_e2e(wl, args.steps * passes, args.warmup, world), world)
    e2e_value = job_throughput(wl.M * passes * args.steps, world, ms_e2e)

    hbm, hbm_src = measured_peaks()
    legs = {}
    if not args.no_skinny:
        skinny = {"workload": "batched decode: M tokens through the 210 projections of 30 "
                              "BitNet-2B4T layers (independent inputs, per-token scales "
                              "U(0.1, 10)), no RMSNorm, bf16 out; weights of the headline",
                  "by_M": {}}
        for Ms in (8, 32, 64):
            sw = SkinnyWorkload(wl, Ms)
            skinny["by_M"][str(Ms)] = sw.measure(reps, rw, world, hbm)
            del sw
        legs["skinny"] = skinny
        fw = FfnChainWorkload(wl)
        legs["ffn_chain"] = fw.measure(reps, rw, world, hbm)
        fw.unfused(wl)
        legs["ffn_chain"]["unfused_gate_up"] = fw.measure_unfused(reps, rw, world)
        del fw
        dc = DecodeChainWorkload(wl)
        legs["decode_chain"] = dc.measure(reps, rw, world, hbm)
        dc.persistent(wl)
        legs["decode_chain_persistent"] = dc.measure_persistent(reps, rw, world, hbm)
        dc.with_attention(wl)
        legs["decode_step_with_attention"] = dc.measure_attention(reps, rw, world, hbm)
        del dc
    if not args.no_skinny:
        att = {"workload": "attention block of one decode token, 2B4T heads (20 query, 5 key/value "
                           "of 128): RoPE of q and of the new k row, grouped-query attention over "
                           "an L-position cache; 30 token-layers per graph", "by_L": {}}
        for Ls in (512, 2048):
            aw = AttentionWorkload(Ls)
            att["by_L"][str(Ls)] = aw.measure(reps, rw, world, hbm)
            del aw
        legs["attention_decode"] = att
    if not args.no_prefill:
        pw = PrefillWorkload()
        legs["prefill"] = pw.measure(reps, rw, world)
        del pw
    if not args.no_comparator:
        cmp_ = Bf16Comparator(wl)
        legs["bf16_comparator"] = cmp_.measure(reps, rw, world)
        del cmp_

    status = wl.B.bitlinear_device_status()
    if status != 0:
        raise RuntimeError("device status %d after the timed region" % status)

    gemv_launch_ms = ms_gemv / reps
    bytes_per_launch = wl.gemv_bytes
    achieved = bytes_per_launch / (gemv_launch_ms / 1000.0) / 1e9
    traffic = recorded_traffic(1)
    variants["token_batch_pass_gbs"] = wl.step_bytes / (ms_step / passes / 1000.0) / 1e9

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "passes_per_step": passes, "ms_per_pass": ms_step / passes,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "int8", "data": "synthetic", "config": workload_config(args, wl),
                "bytes": {"packed_weight_bytes_per_pass": wl.weight_bytes,
                          "algorithmic_bytes_per_pass": wl.step_bytes},
                "roofline": {"bound": "hbm",
                             "kernel": "decode_batch_kernel (the token's 210 projections in one launch)",
                             "achieved": achieved, "peak": hbm, "peak_source": hbm_src,
                             "unit": "GB/s", "frac": achieved / hbm,
                             "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                             "nominal_peak": NOMINAL_HBM_GBS, "traffic": traffic,
                             "launch_us": gemv_launch_ms * 1000.0,
                             "bytes_per_launch": bytes_per_launch, "reps": reps},
                "variants": variants,
                "e2e": {"value": e2e_value, "unit": "tokens/s",
                        "h2d_bytes_per_step": wl.h2d_bytes * passes,
                        "d2h_bytes_per_step": wl.d2h_bytes * passes,
                        "note": "pinned host x in and y out every pass, through the public "
                                "batched forward; two buffer sets, copies on their own "
                                "streams overlap the neighbouring passes' compute"},
                "gpu_launches": wl.launches["token_batch"] * passes * args.steps,
                "clocks": clk.result()}
        line.update(legs)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        wl.graphs.clear()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
