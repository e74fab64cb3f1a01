#!/usr/bin/env python
"""Benchmark of the MXFP8 routed-experts MLP on B200.

One step = one pass of the whole hot path over one batch of synthetic routed
tokens: the DSv3-scale expert layer (E=256, D=7168, F=2048, 16384 tokens
top-8, Zipf(1.0) routing padded to 256) forward and backward -- token and
weight casts, FC1 + SwiGLU + dual quant, FC2, dY casts, FC2 dgrad + dSwiGLU +
dual quant, dW2, dx, dW13 -- plus the standalone SwiGLU + dual quant of
h13 [16384, 2x4096], the bf16 -> MXFP8 cast of the [8192, 7168] transport
payload and its dequantization back to bf16.  After the timed steps the fused
forward is timed against the unfused ("swiglu" plan) forward.

Prints one JSON line.  `value` is the useful (real routed rows) fwd+bwd
TFLOP/s of the expert MLP with inputs resident in HBM; every input is larger
than L2, so no flush is needed between steps.  `e2e` is the same metric
through the public token-major layer API with the step's token inputs copied
from pinned host memory and its results (layer output, dx, router-weight
gradient) copied back to pinned host memory inside the timed region.  `--impl reference` times the CPU oracle on a bounded sample.

Launch: python bench.py [--gpus N --steps K --warmup W]; for N > 1 under
torch.distributed.run (one rank per GPU; each rank runs its own batch, no
collective on the data path: weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

SWIGLU_ROWS, SWIGLU_F = 16384, 4096
CAST_ROWS, CAST_COLS = 8192, 7168
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_SPEC_TFLOPS = 4500.0          # nominal dense MXFP8 tensor peak of one B200 (context beside the measured ones)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def src_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mxfp8_block_scaled_routed_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:12]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded by an ncu capture in profiles/, if the
    capture was taken from the current kernel sources."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"source_hash:\s*([0-9a-f]+)", txt)
    if not m or not h or h.group(1) != src_hash():
        return None
    return float(m.group(1))


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms; only samples taken inside [t0, t1]
    (host wall clock around the timed region) are kept."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(1.0)              # let nvidia-smi start sampling before the timed region

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.3)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        import datetime
        sm, mx_, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                if self.t0 is not None and not (self.t0 - 0.25 <= ts <= self.t1 + 0.25):
                    continue
                sm.append(float(f[2]))
                mx_.append(float(f[3]))
                pw.append(float(f[4]))
            except ValueError:
                continue
            for n, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx_) if mx_ else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_median": float(np.median(pw)) if pw else None}


# ----------------------------------------------------------------------------- the step
class Step:
    """All buffers of one fwd+bwd step, laid out once; run() issues the kernels.

    The sequence is exactly the one mxmoe_quantize_weights + moe_mlp_fwd_q +
    moe_mlp_bwd_q issue (a training step: the weights are quantized once, ROW
    and COL in one pass, and used by both passes), written out call by call so
    each kernel can be bracketed with CUDA events.
    """

    def __init__(self, inp, dev):
        import mxfp8_block_scaled_routed_b200 as mxk
        self.mxk, self.L = mxk, mxk.lib()
        s = inp.spec
        self.E, self.D, self.F = s.E, s.D, s.F
        self.M = M = inp.routing.M
        self.R = inp.routing.R
        self.pad = s.pad
        E, D, F = self.E, self.D, self.F
        u8 = lambda *sh: torch.empty(*sh, dtype=torch.uint8, device=dev)
        bf = lambda *sh: torch.empty(*sh, dtype=torch.bfloat16, device=dev)
        self.x, self.w13, self.w2, self.dy = inp.x, inp.w13, inp.w2, inp.dy
        self.off = torch.from_numpy(inp.routing.offsets).to(dev)
        # token rows of each expert: the weight gradients skip the all-pad K blocks
        counts = np.asarray(inp.routing.counts, dtype=np.int64)
        self.rows = torch.from_numpy(counts.astype(np.int32)).to(dev)
        self.Mw = int(((counts + 127) // 128 * 128).sum())   # rows the weight gradients run over
        self.x_rc, self.x_rs, self.x_cc, self.x_cs = u8(M, D), u8(M * D // 32), u8(D, M), u8(M * D // 32)
        self.qw = self.mxk.make_qweights(E, D, F, dev)
        self.h13 = bf(M, 2 * F)
        self.h_rc, self.h_rs, self.h_cc, self.h_cs = u8(M, F), u8(M * F // 32), u8(F, M), u8(M * F // 32)
        self.y = bf(M, D)
        self.dy_rc, self.dy_rs, self.dy_cc, self.dy_cs = u8(M, D), u8(M * D // 32), u8(D, M), u8(M * D // 32)
        self.g_rc, self.g_rs, self.g_cc, self.g_cs = u8(M, 2 * F), u8(M * 2 * F // 32), u8(2 * F, M), u8(M * 2 * F // 32)
        self.dx, self.dw13, self.dw2 = bf(M, D), bf(E, 2 * F, D), bf(E, D, F)
        # standalone boundary kernels
        self.sw_in = inp.swiglu_h13
        self.sw_rc, self.sw_rs = u8(SWIGLU_ROWS, SWIGLU_F), u8(SWIGLU_ROWS * SWIGLU_F // 32)
        self.sw_cc, self.sw_cs = u8(SWIGLU_F, SWIGLU_ROWS), u8(SWIGLU_ROWS * SWIGLU_F // 32)
        self.c_in = inp.cast_x
        self.c_rc, self.c_rs = u8(CAST_ROWS, CAST_COLS), u8(CAST_ROWS, CAST_COLS // 32)
        self.c_deq = bf(CAST_ROWS, CAST_COLS)
        # dispatcher: routing of the same draw, token rows, router weights, upstream token gradient
        self.T, self.k = s.tokens, s.top_k
        self.topk = torch.from_numpy(inp.routing.topk).to(dev)
        self.x_tok = inp.x_tok
        self.dout = inp.dout_tok
        self.wr = inp.router_w
        self.r_off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.r_row_slot = torch.empty(M, dtype=torch.int32, device=dev)
        self.r_slot_row = torch.empty(self.T * self.k, dtype=torch.int32, device=dev)
        self.r_ws = u8(max(16, int(self.L.mxmoe_route_workspace_size(self.T, self.k, E))))
        self.comb = bf(self.T, D)
        self.dwr = torch.empty(self.T, self.k, dtype=torch.float32, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        self._build()

    def _build(self):
        L, p = self.L, (lambda t: torch.Tensor.data_ptr(t))
        st = self.stream.cuda_stream
        M, D, E, F, pad = self.M, self.D, self.E, self.F, self.pad
        T, k, R = self.T, self.k, self.R
        off = p(self.off)
        q = {k: p(v) for k, v in self.qw.items()}
        self.ops = [
            ("cast_x_dual", "hbm", 4.0625 * M * D,
             lambda: L.mxfp8_quantize(p(self.x), 1, M, D, 3, 1, p(self.x_rc), p(self.x_rs), p(self.x_cc), p(self.x_cs), st)),
            ("cast_w13_dual", "hbm", 4.0625 * E * 2 * F * D,
             lambda: L.mxfp8_quantize(p(self.w13), E, 2 * F, D, 3, 1, q["w13_codes"], q["w13_scales"], q["w13t_codes"],
                                      q["w13t_scales"], st)),
            ("cast_w2_dual", "hbm", 4.0625 * E * D * F,
             lambda: L.mxfp8_quantize(p(self.w2), E, D, F, 3, 1, q["w2_codes"], q["w2_scales"], q["w2t_codes"],
                                      q["w2t_scales"], st)),
            ("fc1_swiglu_quant", "tensor", 2.0 * M * 2 * F * D,
             lambda: L.mxfp8_grouped_gemm_swiglu_quant(p(self.x_rc), p(self.x_rs), M, D, q["w13_codes"], q["w13_scales"], E,
                                                       F, off, pad, p(self.h13), p(self.h_rc), p(self.h_rs), p(self.h_cc),
                                                       p(self.h_cs), st)),
            ("fc2", "tensor", 2.0 * M * D * F,
             lambda: L.mxfp8_grouped_gemm(p(self.h_rc), p(self.h_rs), M, F, q["w2_codes"], q["w2_scales"], E, D, off, pad,
                                          p(self.y), st)),
            ("cast_dy_dual", "hbm", 4.0625 * M * D,
             lambda: L.mxfp8_quantize(p(self.dy), 1, M, D, 3, 1, p(self.dy_rc), p(self.dy_rs), p(self.dy_cc), p(self.dy_cs), st)),
            ("fc2_dgrad_dswiglu_quant", "tensor", 2.0 * M * F * D,
             lambda: L.mxfp8_grouped_gemm_dswiglu_quant(p(self.dy_rc), p(self.dy_rs), M, D, q["w2t_codes"], q["w2t_scales"],
                                                        E, F, off, pad, p(self.h13), p(self.g_rc), p(self.g_rs),
                                                        p(self.g_cc), p(self.g_cs), st)),
            ("wgrad_dw2", "tensor", 2.0 * self.Mw * D * F,
             lambda: L.mxfp8_grouped_gemm_wgrad(p(self.dy_cc), p(self.dy_cs), D, p(self.h_cc), p(self.h_cs), F, M, off,
                                                p(self.rows), E, pad, p(self.dw2), st)),
            ("dgrad_dx", "tensor", 2.0 * M * 2 * F * D,
             lambda: L.mxfp8_grouped_gemm(p(self.g_rc), p(self.g_rs), M, 2 * F, q["w13t_codes"], q["w13t_scales"], E, D, off,
                                          pad, p(self.dx), st)),
            ("wgrad_dw13", "tensor", 2.0 * self.Mw * 2 * F * D,
             lambda: L.mxfp8_grouped_gemm_wgrad(p(self.g_cc), p(self.g_cs), 2 * F, p(self.x_cc), p(self.x_cs), D, M, off,
                                                p(self.rows), E, pad, p(self.dw13), st)),
            ("swiglu_quant_16384x4096", "hbm", 6.0625 * SWIGLU_ROWS * SWIGLU_F,
             lambda: L.mxfp8_swiglu_quant(p(self.sw_in), SWIGLU_ROWS, SWIGLU_F, 3, 1, p(self.sw_rc), p(self.sw_rs),
                                          p(self.sw_cc), p(self.sw_cs), st)),
            ("cast_payload_8192x7168", "hbm", 3.03125 * CAST_ROWS * CAST_COLS,
             lambda: L.mxfp8_quantize(p(self.c_in), 1, CAST_ROWS, CAST_COLS, 1, 0, p(self.c_rc), p(self.c_rs), None, None, st)),
            ("dequant_payload_8192x7168", "hbm", 3.03125 * CAST_ROWS * CAST_COLS,
             lambda: L.mxfp8_dequantize(p(self.c_rc), p(self.c_rs), CAST_ROWS, CAST_COLS, p(self.c_deq), st)),
        ]
        self.mlp_ops = 10
        # dispatcher around the MLP (same routing; m_cap = the padded rows), timed
        # after the step, outside the step's own clock
        self.disp_ops = [
            ("route", "hbm", 4.0 * (3 * T * k + M + 2 * E),
             lambda: L.mxmoe_route(p(self.topk), T, k, E, pad, M, p(self.r_off), p(self.r_row_slot),
                                   p(self.r_slot_row), p(self.r_ws), self.r_ws.numel(), st)),
            ("permute_quant_x_dual", "hbm", 2.0 * R * D + 2.0625 * M * D,
             lambda: L.mxmoe_permute_quant(p(self.x_tok), T, D, p(self.r_row_slot), k, None, M, p(self.r_off) + 4 * E,
                                           3, 1, p(self.x_rc), p(self.x_rs), p(self.x_cc), p(self.x_cs), st)),
            ("permute_quant_dy_weighted", "hbm", 2.0 * R * D + 2.0625 * M * D,
             lambda: L.mxmoe_permute_quant(p(self.dout), T, D, p(self.r_row_slot), k, p(self.wr), M,
                                           p(self.r_off) + 4 * E, 3, 1, p(self.dy_rc), p(self.dy_rs), p(self.dy_cc),
                                           p(self.dy_cs), st)),
            ("combine_y", "hbm", 2.0 * R * D + 2.0 * T * D,
             lambda: L.mxmoe_unpermute_combine(p(self.y), M, D, p(self.r_slot_row), p(self.wr), T, k, p(self.comb), st)),
            ("combine_weight_grad", "hbm", 2.0 * R * D + 2.0 * T * D,
             lambda: L.mxmoe_combine_weight_grad(p(self.dout), p(self.y), M, D, p(self.r_slot_row), T, k, p(self.dwr),
                                                 st)),
        ]
        # the transport payload with E5M2 elements (cast and restore)
        self.e5m2_ops = [
            ("cast_payload_e5m2_8192x7168", "hbm", 3.03125 * CAST_ROWS * CAST_COLS,
             lambda: L.mxfp8_quantize_e5m2(p(self.c_in), 1, CAST_ROWS, CAST_COLS, 1, 0, p(self.c_rc), p(self.c_rs),
                                           None, None, st)),
            ("dequant_payload_e5m2_8192x7168", "hbm", 3.03125 * CAST_ROWS * CAST_COLS,
             lambda: L.mxfp8_dequantize_e5m2(p(self.c_rc), p(self.c_rs), CAST_ROWS, CAST_COLS, p(self.c_deq), st)),
        ]

    def run(self, events=None):
        for i, (name, _, _, fn) in enumerate(self.ops):
            s = fn()
            if s != 0:
                raise RuntimeError(f"{name}: {self.L.mxmoe_last_error_message().decode()}")
            if events is not None:
                events[i + 1].record(self.stream)

    def flops(self, rows):
        return 18.0 * rows * self.D * self.F


# ----------------------------------------------------------------------------- inputs
def make_inputs(workload: str, seed: int, dev):
    import synth
    inp = synth.device_moe_inputs(workload, seed, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed + 7)
    h = torch.randn(SWIGLU_ROWS, 2 * SWIGLU_F, generator=gen, device=dev)
    n = h.numel()
    idx = torch.randperm(n, generator=gen, device=dev)[: n // 100]
    h.view(-1)[idx] *= 100.0
    inp.swiglu_h13 = h.to(torch.bfloat16)
    del h, idx
    inp.cast_x = torch.randn(CAST_ROWS, CAST_COLS, generator=gen, device=dev).to(torch.bfloat16)
    s = inp.spec
    inp.dout_tok = (torch.randn(s.tokens, s.D, generator=gen, device=dev) * s.dy_std).to(torch.bfloat16)
    inp.router_w = torch.from_numpy(synth.router_weights(s.tokens, s.top_k, seed)).to(dev)
    return inp


# ----------------------------------------------------------------------------- CPU baseline (oracle)
def oracle_sample(inp, budget_s=12.0, max_experts=None):
    """Time the CPU oracle (fwd+bwd) on whole experts of the workload, the
    smallest non-empty ones first, until about budget_s of work is done."""
    from oracle import mx
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        cores = os.cpu_count()
    counts = inp.routing.counts
    off = inp.routing.offsets
    order = [int(e) for e in np.argsort(counts) if counts[e] > 0]
    order = order[len(order) // 2:] + order[: len(order) // 2]          # start from the median expert
    f = lambda t: t.float().double().cpu().numpy()
    flops, t_total, rows_done, experts = 0.0, 0.0, 0, []
    for e in order:
        lo, hi = int(off[e]), int(off[e + 1])
        x, dy = f(inp.x[lo:hi]), f(inp.dy[lo:hi])
        w13, w2 = f(inp.w13[e]), f(inp.w2[e])
        t0 = time.perf_counter()
        r = mx.expert_fwd(x, w13, w2)
        mx.expert_bwd(dy, r, x, w13, w2)
        t_total += time.perf_counter() - t0
        flops += 18.0 * int(counts[e]) * inp.spec.D * inp.spec.F
        rows_done += int(counts[e])
        experts.append(e)
        if t_total >= budget_s or (max_experts and len(experts) >= max_experts):
            break
    return dict(value=flops / t_total / 1e12, unit="TFLOP/s", cores=int(cores), kind="oracle",
                sample=f"fwd+bwd of {len(experts)} whole expert(s) ({rows_done} real rows) of the "
                       f"{inp.spec.name} layer, float64 numpy, {t_total:.1f} s"), t_total


# ----------------------------------------------------------------------------- main
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.distributed.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                             timeout=datetime.timedelta(seconds=600))
    return world, rank, local


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    dev = device if device is not None else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Replicas: every rank processes its own batch; the job's throughput is
    all ranks' work over the slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def config_dict(spec, inp, extra=None):
    d = {"workload": f"{spec.name}: E={spec.E} D={spec.D} F={spec.F} tokens={spec.tokens} top{spec.top_k} "
                     f"Zipf({spec.zipf_s}) pad {spec.pad}, fwd+bwd; + SwiGLU quant 16384x2x4096 + cast 8192x7168",
         "tokens": spec.tokens, "top_k": spec.top_k, "padded_rows": int(inp.routing.M), "real_rows": int(inp.routing.R),
         "l2": "inputs larger than L2 (x, dy, weights >> 126 MB); no flush needed"}
    if extra:
        d.update(extra)
    return d


def run_reference(args, world, rank):
    import synth
    if rank != 0:
        return 0
    spec = synth.SPECS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = synth.device_moe_inputs(spec, args.seed, device=dev)
    for _ in range(args.warmup):
        oracle_sample(inp, budget_s=2.0, max_experts=1)
    times, vals = [], []
    cpu = None
    for _ in range(args.steps):
        cpu, t = oracle_sample(inp, budget_s=4.0)
        times.append(t)
        vals.append(cpu["value"])
    v = float(np.mean(vals))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * float(np.mean(times)),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(spec, inp),
            "cpu_baseline": dict(cpu, value=v),
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


METRIC = "MoE expert-MLP MXFP8 fwd+bwd TFLOP/s (useful rows); SwiGLU+quant GB/s vs HBM peak"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="dsv3", choices=["dsv3", "dsv3_16b", "dsv3_slice", "tiny"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        # rank 0 alone times the oracle; no process group, no collectives
        return run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
    world, rank, local = dist_setup(args)

    assert torch.cuda.is_available(), "bench.py needs a GPU"
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import mxfp8_block_scaled_routed_b200 as mxk
    import synth
    spec = synth.SPECS[args.workload]
    inp = make_inputs(args.workload, args.seed + rank, dev)
    step = Step(inp, dev)
    n_ops = len(step.ops)

    # warm-up (at least 3 steps)
    args.warmup = max(args.warmup, 3)
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    if mxk.device_error() != 0:
        raise RuntimeError("device error during warm-up")

    # timed region: K steps, CUDA events around every kernel on the launch stream
    gpu_index = local
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            gpu_index = int(vis.split(",")[local])
        except ValueError:
            pass
    clocks = ClockSampler(gpu_index)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ops + 1)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    clocks.mark_start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(step.stream)
    for k in range(args.steps):
        evs[k][0].record(step.stream)
        step.run(evs[k])
    t_end.record(step.stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    ms_total = t_start.elapsed_time(t_end)
    if mxk.device_error() != 0:
        raise RuntimeError("device error during the timed region")
    per = np.array([[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(n_ops)] for k in range(args.steps)])
    mean_ms = per.mean(axis=0)
    ms_step = max_over_ranks(ms_total / args.steps, dev)

    peaks, peak_src = load_peaks()
    fp8_sus = 2.0 * peaks["bf16_tflops_sustained"]     # MXFP8 dense = 2 x bf16 (nominal 4.5 / 2.25 PF)
    fp8_burst = 2.0 * peaks["bf16_tflops"]
    hbm = peaks["hbm_gbs"]
    kernels = {}
    for (name, bound, work, _), ms in zip(step.ops, mean_ms):
        if bound == "tensor":
            ach = work / (ms * 1e-3) / 1e12
            kernels[name] = {"ms": round(float(ms), 4), "TFLOP/s": round(ach, 1), "frac": round(ach / fp8_sus, 3),
                             "frac_burst": round(ach / fp8_burst, 3), "frac_spec": round(ach / FP8_SPEC_TFLOPS, 3)}
        else:
            ach = work / (ms * 1e-3) / 1e9
            kernels[name] = {"ms": round(float(ms), 4), "GB/s": round(ach, 1), "frac": round(ach / hbm, 3)}
    mlp_ms = float(mean_ms[: step.mlp_ops].sum())
    cast_w_ms = float(sum(mean_ms[i] for i, (n, *_r) in enumerate(step.ops) if n.startswith("cast_w")))
    useful = step.flops(step.R)
    # executed: the forward and the dgrad GEMMs over the padded rows, the weight
    # gradients over each expert's rows rounded up to 128 (12 + 6 of the 18 M.D.F)
    executed = step.flops(step.M) * 12.0 / 18.0 + step.flops(step.Mw) * 6.0 / 18.0
    value = whole_job_tflops(useful, world, ms_step)
    fwd_ms = float(mean_ms[[0, 3, 4]].sum())   # x cast, FC1, FC2 (weights already quantized)

    # fused vs unfused forward (the pages' comparison), same inputs and weights
    def fwd_fused():
        step.ops[0][3]()
        step.ops[3][3]()
        step.ops[4][3]()

    def fwd_unfused():
        L, p, st = step.L, (lambda t: t.data_ptr()), step.stream.cuda_stream
        q = {k: p(v) for k, v in step.qw.items()}
        M, D, E, F, pad, off = step.M, step.D, step.E, step.F, step.pad, p(step.off)
        step.ops[0][3]()
        L.mxfp8_grouped_gemm(p(step.x_rc), p(step.x_rs), M, D, q["w13_codes"], q["w13_scales"], E, 2 * F, off, pad,
                             p(step.h13), st)
        L.mxfp8_swiglu_quant(p(step.h13), M, F, 3, 1, p(step.h_rc), p(step.h_rs), p(step.h_cc), p(step.h_cs), st)
        step.ops[4][3]()

    def time_it(fn, n=5):
        for _ in range(2):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(step.stream)
        for _ in range(n):
            fn()
        e1.record(step.stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    ms_fused, ms_unfused = time_it(fwd_fused), time_it(fwd_unfused)
    fused_vs_unfused = {"fused_fwd_ms": round(ms_fused, 3), "unfused_fwd_ms": round(ms_unfused, 3),
                        "fused_speedup": round(ms_unfused / ms_fused, 4),
                        "what": "x cast + FC1 (+SwiGLU + dual quant fused in the epilogue) + FC2, vs x cast + FC1 "
                                "to bf16 h13 + standalone SwiGLU + dual quant + FC2; same padding (pad-matched)"}

    # kernels outside the step (the token dispatcher, the E5M2 transport
    # variant): each timed alone over n launches
    def time_group(ops):
        res = {}
        for name, bound, work, fn in ops:
            if fn() != 0:
                raise RuntimeError(f"{name}: {step.L.mxmoe_last_error_message().decode()}")
            ms = time_it(fn, n=10)
            ach = work / (ms * 1e-3) / 1e9
            res[name] = {"ms": round(ms, 4), "GB/s": round(ach, 1), "frac": round(ach / hbm, 3)}
        if mxk.device_error() != 0:
            raise RuntimeError("device error outside the step")
        return res

    outside_step = {"dispatcher": time_group(step.disp_ops), "e5m2_transport": time_group(step.e5m2_ops)}

    # dominant kernel and its roofline
    imax = int(np.argmax(mean_ms[: step.mlp_ops]))
    dname, dbound, dwork, _ = step.ops[imax]
    dms = float(mean_ms[imax])
    if dbound == "tensor":
        ach = dwork / (dms * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": dname, "achieved": round(ach, 1), "peak": round(fp8_sus, 1),
                "unit": "TFLOP/s", "frac": round(ach / fp8_sus, 3), "frac_burst": round(ach / fp8_burst, 3),
                "frac_spec": round(ach / FP8_SPEC_TFLOPS, 3),
                "peak_source": f"{peak_src} bf16 sustained x 2 (MXFP8 nominal ratio)",
                "traffic": ncu_traffic(dname, args.workload)}
    else:
        ach = dwork / (dms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dname, "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(ach / hbm, 3), "peak_source": f"{peak_src} hbm_gbs",
                "traffic": ncu_traffic(dname, args.workload)}

    # end to end through the public token-major layer API, host buffers: the
    # step's inputs (token rows, routing, router weights, upstream gradient)
    # are copied from pinned host memory every step and the results copied
    # back; weights stay resident
    e2e = None
    if not args.no_e2e:
        T, k = spec.tokens, spec.top_k
        host = [inp.x_tok.cpu().pin_memory(), torch.from_numpy(inp.routing.topk).pin_memory(),
                inp.router_w.cpu().pin_memory(), inp.dout_tok.cpu().pin_memory()]
        # two device slots for the step inputs and for its outputs: the copy of
        # step i+1's inputs (H2D stream) and the read-back of step i's outputs
        # (D2H stream) overlap the neighbouring steps' compute; every step's
        # copies are inside the timed region
        slots = [[torch.empty_like(h, device=dev) for h in host] for _ in range(2)]
        lsaved = mxk.make_layer_saved(T, k, spec.D, spec.E, spec.F, spec.pad, dev)
        ws_f = torch.empty(mxk.layer_workspace_bytes(T, k, spec.D, spec.E, spec.F, spec.pad, 1), dtype=torch.uint8,
                           device=dev)
        ws_b = torch.empty(mxk.layer_workspace_bytes(T, k, spec.D, spec.E, spec.F, spec.pad, 2), dtype=torch.uint8,
                           device=dev)
        outs = [[torch.empty(T, spec.D, dtype=torch.bfloat16, device=dev),
                 torch.empty(T, spec.D, dtype=torch.bfloat16, device=dev),
                 torch.empty(T, k, dtype=torch.float32, device=dev)] for _ in range(2)]
        # the step's results in pinned host memory: layer output, dx, router-weight gradient
        res_h = [torch.empty(T, spec.D, dtype=torch.bfloat16).pin_memory(),
                 torch.empty(T, spec.D, dtype=torch.bfloat16).pin_memory(),
                 torch.empty(T, k, dtype=torch.float32).pin_memory()]
        comp = torch.cuda.current_stream(dev)
        copy_s = torch.cuda.Stream(dev)
        d2h_s = torch.cuda.Stream(dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        used = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        read = [torch.cuda.Event() for _ in range(2)]

        def h2d(i):
            sl = i % 2
            with torch.cuda.stream(copy_s):
                if i >= 2:
                    copy_s.wait_event(used[sl])        # step i-2 finished reading this slot
                for d, h in zip(slots[sl], host):
                    d.copy_(h, non_blocking=True)
                copied[sl].record(copy_s)

        def compute(i):
            sl = i % 2
            comp.wait_event(copied[sl])
            if i >= 2:
                comp.wait_event(read[sl])              # step i-2's results have left this slot
            x_d, tk_d, w_d, do_d = slots[sl]
            out_d, dx_d, dwr_d = outs[sl]
            mxk.mxmoe_quantize_weights(step.w13, step.w2, qw=step.qw)
            mxk.moe_layer_fwd_q(x_d, tk_d, w_d, step.qw, spec.pad, out=out_d, saved=lsaved, workspace=ws_f)
            mxk.moe_layer_bwd_q(do_d, w_d, step.qw, lsaved, spec.pad, dx=dx_d, dw13=step.dw13, dw2=step.dw2,
                                dweights=dwr_d, workspace=ws_b)
            used[sl].record(comp)
            computed[sl].record(comp)

        def d2h(i):
            sl = i % 2
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(computed[sl])
                for h, d in zip(res_h, outs[sl]):
                    h.copy_(d, non_blocking=True)
                read[sl].record(d2h_s)

        def run(nsteps):
            h2d(0)
            for i in range(nsteps):
                if i + 1 < nsteps:
                    h2d(i + 1)
                compute(i)
                d2h(i)

        run(2)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(comp)
        copy_s.wait_stream(comp)                        # the first copies start inside the timed region
        d2h_s.wait_stream(comp)
        run(args.steps)
        comp.wait_stream(copy_s)
        comp.wait_stream(d2h_s)                         # the last read-back ends inside the timed region
        b.record(comp)
        torch.cuda.synchronize()
        ms = max_over_ranks(a.elapsed_time(b) / args.steps, dev)
        h2d_bytes = sum(h.numel() * h.element_size() for h in host)
        d2h_bytes = sum(h.numel() * h.element_size() for h in res_h)
        e2e = {"value": round(whole_job_tflops(useful, world, ms), 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d_bytes), "d2h_bytes_per_step": int(d2h_bytes),
               "ms_per_step": round(ms, 3),
               "how": "public C-ABI token-major layer (mxmoe_quantize_weights, moe_layer_fwd_q: route + gather/cast + "
                      "MLP + weighted combine, moe_layer_bwd_q: weighted gather/cast + MLP backward + unpermute + "
                      "router-weight gradient); token rows, top-k ids, router weights and the upstream gradient "
                      "copied from pinned host memory every step, and the layer output, dx and the router-weight "
                      "gradient copied back to pinned host memory every step, on two copy streams overlapping the "
                      "neighbouring steps' compute; expert-weight gradients stay on the device"}
        if mxk.device_error() != 0:
            raise RuntimeError("device error during the e2e run")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, _ = oracle_sample(inp)
        cpu["value"] = round(cpu["value"], 6)

    sw = kernels["swiglu_quant_16384x4096"]
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "mxfp8 (e4m3 + e8m0 scales), fp32 accumulate, bf16 io",
        "data": "synthetic (seeded routing, device-drawn bf16 activations and weights)",
        "config": config_dict(spec, inp, {"parallelism": f"replicas x{world} (no data-path collective)"}),
        "fwd_bwd_useful_tflops": round(value, 2),
        "fwd_bwd_executed_tflops": round(whole_job_tflops(executed, world, ms_step), 2),
        "mlp_ms": round(mlp_ms, 3),
        "mlp_no_weight_cast_tflops": round(useful / ((mlp_ms - cast_w_ms) * 1e-3) / 1e12, 2),
        "fwd_useful_tflops_prequantized_weights": round(6.0 * step.R * spec.D * spec.F / (fwd_ms * 1e-3) / 1e12, 2),
        "swiglu_quant_gbs": sw["GB/s"], "swiglu_quant_frac_hbm": sw["frac"],
        "kernel_peaks": {"hbm_gbs": hbm, "mxfp8_tflops_sustained": round(fp8_sus, 1),
                         "mxfp8_tflops_burst": round(fp8_burst, 1), "mxfp8_tflops_spec": FP8_SPEC_TFLOPS,
                         "source": f"{peak_src}: HBM copy; MXFP8 = 2 x the cuBLAS bf16 figure (frac: sustained, "
                                   "frac_burst: burst), frac_spec: the nominal 4.5 PFLOP/s"},
        "kernels": kernels, "fused_vs_unfused": fused_vs_unfused, "outside_step": outside_step, "roofline": roof, "clocks": clk,
        "gpu_launches": n_ops * args.steps,
        "e2e": e2e, "cpu_baseline": cpu, "source_hash": src_hash(),
    }
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
