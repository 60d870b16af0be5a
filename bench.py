#!/usr/bin/env python
"""Throughput of the E2-TTT chunk-parallel closed-form fast-weight update on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload layer_1p3b_2k] [--mode fwd|train]

One step = one e2ttt_chunk_scan_fwd call (mode train: forward then
e2ttt_chunk_scan_bwd) over the whole workload, inputs resident in HBM. The
default workload is the 1.3B-shaped layer (B=4, H=8 heads of 256, SwiGLU fast
hidden 512, T=2048, C=512) with seeded synthetic inputs. The working set
(inputs, fp32 state, workspace) is larger than the 126 MB L2, so no flush is
needed between steps. Time is taken with CUDA events on the launch stream,
max over ranks. Prints one JSON line (rank 0).

N > 1 (torchrun, one process per GPU): every rank runs its own replica of the
workload (independent batch rows, no collective on the data path; weak
scaling); the only collectives are the timing barrier and the max over ranks.

--impl reference: the fp64 CPU oracle (closed form) on a bounded sample of the
same workload, timed on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import e2ttt_inputs as gen  # noqa: E402

METRIC = "E2-TTT layer tokens/sec (fwd, fwd+bwd) at T=2K/16K; % of bf16 TC roofline"
UNIT = "tokens/s"
_CSRC = "test_weight_layers_chunk_b200/csrc/"
# the sources a kernel's recorded ncu traffic depends on, by kernel-name prefix
# (its translation unit and every header that unit compiles)
_SHARED = [_CSRC + "common.cuh", _CSRC + "state.cuh", _CSRC + "paths.h", _CSRC + "trace.h"]
KERNEL_SOURCES = {"tcb_": [_CSRC + "tc_gemm.cuh", _CSRC + "tc_gemm2.cuh", _CSRC + "tc_bwd.cu"] + _SHARED,
                  "tc_": [_CSRC + "tc_gemm.cuh", _CSRC + "tc_gemm2.cuh", _CSRC + "tc_gemm_pair.cuh",
                          _CSRC + "tc_fwd.cu"] + _SHARED,
                  "": [_CSRC + "scan.cu", _CSRC + "simt.cuh", _CSRC + "simt_fwd.cu", _CSRC + "bwd.cu"] + _SHARED}


# ----------------------------------------------------------------- algorithmic work
def phase_flops_per_token_head(w) -> dict:
    """Algorithmic FLOPs per token and head of each forward GEMM phase."""
    dk, dv, dh = w.d_k, w.d_v, w.d_h
    if w.kind == gen.LINEAR:
        return {"tc_g1_linear_out_e": 4 * dk * dv, "tc_g4_aggregate_state": 4 * dv * dk}
    if w.kind == gen.GELU:
        return {"tc_g1_gelu": 4 * dk * dh,             # [q; k] x W1^T
                "tc_g2_y_out_e": 4 * dh * dv,          # [A_q; A_k] x W2^T
                "tc_g3_gelu_dh": 2 * dv * dh,          # E x W2
                "tc_g4_aggregate_state": 4 * dh * dk + 4 * dv * dh}  # two aggregations x 2 matrices
    return {"tc_g1_h_act": 8 * dk * dh,            # [q; k] x [W1; W3]^T
            "tc_g2_y_out_e": 4 * dh * dv,          # [A_q; A_k] x W2^T
            "tc_g3_da_dh": 2 * dv * dh,            # E x W2
            "tc_g4_aggregate_state": 8 * dh * dk + 4 * dv * dh}  # two aggregations x 3 matrices


# Backward kernels of the CUDA-core path (fp32 FMA), algorithmic FLOPs per token
# and head (SwiGLU, d_k = d_v); bwd_h / bwd_residual / bwd_da recompute the
# forward internals at the chunk-start weights.
BWD_SIMT_FLOPS = {"bwd_dk": 12, "bwd_dw2": 6, "bwd_dir_w13": 8, "bwd_h": 8, "bwd_dw13": 8,
                  "bwd_dir_w2": 4, "bwd_residual": 2, "bwd_ub_dir": 4, "bwd_dq": 4, "bwd_eb": 2,
                  "bwd_q_rows": 2, "bwd_da": 2, "bwd_ub_eb": 2}


# Backward GEMM launches of the tensor-core path, FLOPs per token and head in units
# of d d_h (SwiGLU, d_k = d_v = d): 52 for the adjoint plus 14 of recomputation:
# H, E and du at the chunk-start weights (r1 8, r2 2, the du half of r3_q1 2) and
# du once more in e5 (its second accumulator). Four launches carry two phases
# each: r3_q1 (du, dH; the query rows' h1b, h3b), d1_d2 (the directional
# products with the state adjoints), e3_dk1 (ub, dub; dk part 1), dk2_dq (dk, dq).
# With the forward's E and dH saved (save_acts) r2_e and r3_q1 do not run and Q1
# runs alone (q1_hbq): 52 + 10.
TC_BWD_FLOPS = {"tcb_r1_h": 8, "tcb_r2_e": 2, "tcb_r3_q1": 4, "tcb_d1_d2": 12,
                "tcb_e3_dk1": 12, "tcb_e4_eb": 2, "tcb_e5_hb": 4, "tcb_dk2_dq": 8, "tcb_dw": 14,
                "tcb_q1_hbq": 2}


def kernel_work(w, has_m0: bool) -> dict:
    """Work of one launch of each kernel: (FLOPs, algorithmic bytes,
    implementation bytes). One launch covers one chunk of every head (the prep
    kernels and K1: the whole call).

    Algorithmic bytes are the method's compulsory traffic: q, k, v and out once
    in the activation dtype, the three gates once, W0 and M0 read and W_end and
    M_end written once per call (fp32), each charged to the kernel that moves it
    (q, k to the first GEMM phase, v, out to the phase that forms out and E, the
    state to the aggregation phase, one chunk's share per launch). K1 is rated
    as an operator of its own: gates in, a and b out, chunk scalars out. Traffic
    of intermediates (activations, residuals, scaled operand copies, bf16 state
    copies) and the per-chunk round trip of the state through HBM are
    implementation overhead: they are in the implementation bytes (every operand
    read once and every result written once, the state traffic averaged over the
    chunks of a call), never in the algorithmic ones."""
    BH, C, T, NC = w.B * w.H, w.C, w.T, -(-w.T // w.C)
    dk, dv, dh = w.d_k, w.d_v, w.d_h
    k1 = 20.0 * BH * T + 12.0 * BH * NC
    out = {"k1_chunk_coeffs": (0.0, k1, k1),
           "k1_chunk_coeffs_bwd": (0.0, 32.0 * BH * T, 32.0 * BH * T)}
    if w.kind == gen.LINEAR:
        return out
    nf = 2 if w.kind == gen.SWIGLU else 1            # activation factors per hidden unit
    S13, S2 = nf * dh * dk, dv * dh
    S = S13 + S2
    N, Mk, Mv = C * dh, C * dk, C * dv
    st_read = (4 + 4 * has_m0) + 8 * (NC - 1)       # per state element, summed over chunks
    st_write = 8 * NC + 2 * (NC - 1)
    fl = phase_flops_per_token_head(w)
    g1, g3 = ("tc_g1_h_act", "tc_g3_da_dh") if nf == 2 else ("tc_g1_gelu", "tc_g3_gelu_dh")
    state_alg = 16.0 * S / NC                        # W0, M0 in, W_end, M_end out, once per call
    per_head = {
        g1: (fl[g1] * C, 2 * 2 * Mk, 2 * (2 * Mk + S13 + 2 * N + nf * N)),
        "tc_g2_y_out_e": (fl["tc_g2_y_out_e"] * C, 2 * 2 * Mv, 2 * (2 * N + S2 + Mv + 4 * Mv)),
        g3: (fl[g3] * C, 0.0, 2 * (Mv + S2 + nf * N + nf * N)),
        "tc_g4_aggregate_state": (fl["tc_g4_aggregate_state"] * C, state_alg,
                                  2 * (nf * N + 2 * Mk + 2 * Mv + N) + S * (st_read + st_write) / NC),
    }
    if dk == dv and nf == 2:
        dd = dk * dh
        b = {"tcb_r1_h": 4 * Mk + 2 * S13 + 12 * N, "tcb_r2_e": 2 * N + 2 * S2 + 4 * Mv,
             "tcb_r3_q1": (2 * Mv + 2 * S2 + 8 * N) + (2 * Mv + 2 * S2 + 8 * N),
             "tcb_q1_hbq": 2 * Mv + 2 * S2 + 8 * N,
             "tcb_d1_d2": (2 * Mk + 4 * S13 + 12 * N) + (2 * N + 4 * S2 + 6 * Mv),
             "tcb_e3_dk1": (2 * Mv + 4 * S2 + 18 * N) + (4 * N + 4 * S13 + 4 * Mk),
             "tcb_e4_eb": 2 * N + 2 * S2 + 8 * Mv, "tcb_e5_hb": 4 * Mv + 2 * S2 + 20 * N,
             "tcb_dk2_dq": (4 * N + 2 * S13 + 6 * Mk) + (4 * N + 2 * S13 + 2 * Mk),
             "tcb_dw": 14 * N + 4 * Mk + 6 * Mv + 8 * S}
        # algorithmic bytes of the backward: q, k, v, dout read and dq, dk, dv
        # written once (bf16); the saved chunk-start states read once (the shadow
        # pass); dW0, dM0 written once per call (the dW phase, one chunk's share)
        alg = {"tcb_r1_h": 2 * 2 * Mk, "tcb_r2_e": 2 * Mv, "tcb_r3_q1": 2 * Mv, "tcb_q1_hbq": 2 * Mv,
               "tcb_e4_eb": 2 * Mv, "tcb_dk2_dq": 2 * 2 * Mk, "tcb_dw": 8.0 * S / NC}
        for n, by in b.items():
            per_head[n] = (TC_BWD_FLOPS[n] * dd * C, float(alg.get(n, 0.0)), by)
        per_head["tcb_shadow"] = (0.0, 8.0 * S, 26.0 * S)
    out.update({n: (f * BH, a * BH, by * BH) for n, (f, a, by) in per_head.items()})
    # the persistent forward: every chunk's four GEMM phases in one launch
    phases = (g1, "tc_g2_y_out_e", g3, "tc_g4_aggregate_state")
    out["tc_fwd_persistent"] = tuple(NC * sum(out[n][i] for n in phases) for i in range(3))
    # the fused G1 + G2 launch (SwiGLU, opt-in): both phases' work; its bytes
    # drop the query rows' u, which stays on chip (written once, read once)
    u_query = 2.0 * 2 * BH * C * dh
    out["tc_ff12_h_y"] = (out[g1][0] + out["tc_g2_y_out_e"][0], out[g1][1] + out["tc_g2_y_out_e"][1],
                          out[g1][2] + out["tc_g2_y_out_e"][2] - u_query)
    out["tc_shadow_init"] = (0.0, 0.0, 6.0 * S * BH)
    out["tc_scale_keys"] = (0.0, 0.0, 6.0 * T * dk * BH)
    # the two in one launch (the scaled keys only for the MLP fast weights)
    out["tc_prep"] = (0.0, 0.0, out["tc_shadow_init"][2] + (out["tc_scale_keys"][2] if w.kind != gen.LINEAR else 0.0))
    return out


def roofline_of(flops: float, alg_bytes: float, seconds: float, peaks: dict) -> dict:
    """Bound and fraction of one launch from its algorithmic work: the slower of
    FLOPs at the measured bf16 peak and bytes at the measured copy bandwidth
    decides the bound; the fraction is the achieved rate over that peak."""
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = alg_bytes / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        a = flops / seconds / 1e12
        return {"bound": "tensor", "achieved": a, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": a / peaks["bf16_tflops"], "algorithmic_per_launch": flops,
                "peak_source": peaks["source"] + " (burst bf16 GEMM)"}
    a = alg_bytes / seconds / 1e9
    return {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": a / peaks["hbm_gbs"], "algorithmic_per_launch": alg_bytes,
            "peak_source": peaks["source"] + " (copy bandwidth)"}


def fwd_flops(w) -> float:
    return float(sum(phase_flops_per_token_head(w).values())) * w.B * w.H * w.T


def train_flops(w) -> float:
    """Forward plus backward: the backward's algorithmic FLOPs are twice the
    forward's (SwiGLU, d_k = d_v = d: 26 + 52 d d_h per token and head; the same
    ratio is taken for the GELU MLP); the backward's recomputation of the forward
    is not counted."""
    return 3.0 * fwd_flops(w)


def fp32_fma_peak_tflops(sm_mhz: float) -> float:
    """CUDA-core fp32 peak from unit counts: 148 SMs x 128 FP32 lanes x 2 FLOP
    per FMA x clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def algorithmic_bytes(w) -> float:
    """q, k, v, out once (act dtype), gates, W0/M0 in and W_end/M_end out (fp32)."""
    es = 2 if w.act == gen.BF16 else 4
    toks = w.B * w.H * w.T
    return toks * (2 * w.d_k + 2 * w.d_v) * es + toks * 12 + 4 * w.B * w.H * w.state_elems * 4


# ----------------------------------------------------------------- environment
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity for one rank)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def kernel_source_sha(kernel: str) -> str:
    prefix = next(p for p in KERNEL_SOURCES if kernel.startswith(p))
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[prefix]:
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel, if it
    was taken on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", txt)
    tb = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not sha or not tb or sha.group(1) != kernel_source_sha(kernel):
        return None
    return float(tb.group(1))


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------- CPU oracle timing
def _pool_threads() -> int:
    """Threads of the BLAS / OpenMP pools the oracle's numpy calls run on."""
    from threadpoolctl import threadpool_info
    return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])


def oracle_sample(w, x, budget_s: float, routine: str = "closed", max_heads=None,
                  max_tokens=None):
    """Run one fp64 oracle routine head by head until `budget_s` is spent.
    routine "closed": closed_fwd over whole heads; "seq": the per-token
    recurrence seq_fwd over the first `max_tokens` tokens of each head (a
    bounded sample: it is about 30 times slower). Returns (layer tokens
    processed, seconds, heads, token count per head)."""
    import oracle as O
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    if max_heads:
        heads = heads[:max_heads]
    T = min(w.T, max_tokens) if max_tokens else w.T
    done = 0
    t0 = time.perf_counter()
    for (b, h) in heads:
        if routine == "closed":
            O.closed_fwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"],
                         x["M0"], w.C, d_h=w.d_h, loss=w.loss, heads=[(b, h)])
        else:
            sl = lambda a: a[b:b + 1, h:h + 1, :T]
            O.seq_fwd(w.kind, sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["lr"]), sl(x["mom"]),
                      sl(x["decay"]), x["W0"][b:b + 1, h:h + 1], x["M0"][b:b + 1, h:h + 1], w.C,
                      d_h=w.d_h, loss=w.loss)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    # layer tokens = token-heads / H (a layer token carries all H heads)
    return done * T / w.H, dt, done, T


def cpu_baselines(w, x, budget_s: float) -> dict:
    """The fp64 oracle on the host cores: closed_fwd and the per-token seq_fwd,
    each single-threaded and with every core, over bounded samples of the
    workload. The line's value is closed_fwd with every core (the fastest)."""
    cores = os.cpu_count() or 1
    runs = []
    from threadpoolctl import threadpool_limits
    for routine, limit in (("closed", None), ("closed", 1), ("seq", None), ("seq", 1)):
        with threadpool_limits(limits=limit):
            n = _pool_threads()
            if routine == "closed":
                tok, dt, nh, T = oracle_sample(w, x, budget_s, "closed")
                sample = f"closed_fwd on {nh} of {w.B * w.H} heads x {T} tokens ({dt:.1f} s)"
            else:
                tok, dt, nh, T = oracle_sample(w, x, budget_s / 2, "seq", max_heads=1,
                                               max_tokens=min(w.T, w.C))
                sample = f"seq_fwd on {nh} head x its first {T} tokens ({dt:.1f} s)"
        runs.append({"routine": routine + "_fwd", "threads": n, "value": tok / dt, "unit": UNIT,
                     "sample": sample})
    best = runs[0]
    return {"value": best["value"], "unit": UNIT, "cores": best["threads"], "kind": "oracle",
            "sample": best["sample"] + f"; host has {cores} cores", "runs": runs}


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    x = gen.generate(w)
    for _ in range(args.warmup):
        oracle_sample(w, x, 0.0, max_heads=1)
    tok = 0.0
    t0 = time.perf_counter()
    threads = _pool_threads()
    for _ in range(args.steps):
        t, _, _, _ = oracle_sample(w, x, 0.0, max_heads=1)
        tok += t
    dt = time.perf_counter() - t0
    v = tok / dt
    sample = f"closed-form fp64 oracle, 1 of {w.B * w.H} heads x {w.T} tokens per step"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w, args),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))


KIND_NAMES = {gen.LINEAR: "linear", gen.SWIGLU: "swiglu", gen.GELU: "gelu_mlp"}


def config_dict(w, args):
    return {"workload": w.name, "kind": KIND_NAMES[w.kind],
            "B": w.B, "H": w.H, "d_k": w.d_k, "d_v": w.d_v, "d_h": w.d_h, "T": w.T, "C": w.C,
            "global_batch": w.B * args.gpus, "seq_len": w.T, "mode": args.mode,
            **({"save_acts": True} if args.mode == "train" else {}),
            "parallelism": f"replicas{args.gpus}" if args.gpus > 1 else "single",
            "l2": "working set larger than L2 (no flush)"}


def capture_graph(torch, dev, stream, fn):
    """One step (every launch of the C-ABI calls) captured as a CUDA graph, for
    replay without the host-side launch cost. fn(st) must launch on st."""
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        fn(cap)
    cap.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        fn(cap)
    torch.cuda.synchronize(dev)
    return g


# ----------------------------------------------------------------- extra lines
def _timed(torch, stream, fn, steps):
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(steps):
        fn()
    ev1.record(stream)
    torch.cuda.synchronize()
    return ev0.elapsed_time(ev1) / steps


def measure_k1_large(E, torch, dev, stream, reps: int = 20) -> dict:
    """K1 alone on B*H*T = 2^26 token-heads (64 heads x 2^20 tokens, C = 512), large
    enough that its bandwidth means something: 12 B of gates in and 8 B of a, b
    out per token-head plus 12 B of chunk scalars per chunk, once each. Gates are
    drawn on the device in the workload's ranges (lr U(0.01, 0.1), momentum
    U(0.8, 0.99), decay U(0.95, 1)); CUDA events on the launching stream, after
    warm-up; the 1.3 GB touched per launch is ten times L2."""
    BH, T, C = 64, 1 << 20, 512
    g = torch.Generator(device=dev).manual_seed(26)
    u = lambda lo, hi: lo + (hi - lo) * torch.rand((BH, T), generator=g, device=dev)
    lr, mom, decay = u(0.01, 0.1), u(0.8, 0.99), u(0.95, 1.0)
    a, b = torch.empty_like(lr), torch.empty_like(lr)
    nc = T // C
    sc = torch.empty((3, BH, nc), device=dev)
    shape = E.make_shape(BH, 1, T, C, 1, 1, 0, E.LINEAR, E.F32)
    run = lambda: E.e2ttt_chunk_coeffs(shape, lr, mom, decay, a, b, sc, stream=stream)
    for _ in range(3):
        run()
    ms = _timed(torch, stream, run, reps)
    by = 20.0 * BH * T + 12.0 * BH * nc
    gbs = by / (ms / 1e3) / 1e9
    peak = measured_peaks()
    out = {"token_heads": BH * T, "us_per_launch": ms * 1e3, "bytes_per_launch": by, "gbs": gbs,
           "frac": gbs / peak["hbm_gbs"], "peak_source": peak["source"] + " (copy bandwidth)"}
    del lr, mom, decay, a, b, sc
    torch.cuda.empty_cache()
    return out


def measure_extras(E, torch, dev, stream, args):
    """The metric's other operating points, device-timed like the main line:
    the forward of the tiny linear workload (fp32, CUDA cores) and of the d = 128
    SwiGLU workload (both latency-bound), forward at T = 16K (the 8x length-extrapolation layer), forward+backward at
    T = 2K (the training workload), the forward at T = 2K of the
    chunk-averaged variant, of the no-momentum mode and of the GELU MLP fast
    weight, and the GELU MLP's forward+backward at T = 2K, each with its own
    warm-up."""
    out = {}
    f = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(dt)
    for name, train, steps, coef, nomom in (("tiny_linear", False, args.extra_steps, 0, 0),
                                            ("swiglu_d128", False, args.extra_steps, 0, 0),
                                            ("layer_1p3b_16k", False, args.extra_steps, 0, 0),
                                            ("train_1p3b_2k", True, max(2, args.extra_steps // 8), 0, 0),
                                            ("layer_1p3b_2k", False, args.extra_steps, 1, 0),
                                            ("layer_1p3b_2k", False, args.extra_steps, 0, 1),
                                            ("layer_1p3b_2k_gelu", False, args.extra_steps, 0, 0),
                                            ("layer_1p3b_2k_gelu", True, max(2, args.extra_steps // 8), 0, 0)):
        w = gen.BY_NAME[name]
        x = gen.generate(w)
        ad = torch.bfloat16 if w.act == gen.BF16 else torch.float32
        q, k, v = f(x["q"], ad), f(x["k"], ad), f(x["v"], ad)
        lr, mom, decay, W0 = f(x["lr"]), f(x["mom"]), f(x["decay"]), f(x["W0"])
        shape = E.make_shape(w.B, w.H, w.T, w.C, w.d_k, w.d_v, w.d_h, w.kind, w.act, w.loss,
                             coef=coef, momentum=nomom,
                             save_acts=E.SAVE_ACTS if train and w.kind != gen.LINEAR else E.RECOMPUTE_ACTS)
        outb, We, Me = torch.empty_like(v), torch.empty_like(W0), torch.empty_like(W0)
        saved = E.saved_states(shape, dev) if train else None
        ws = E.workspace(shape, False, dev)
        if train:
            dout = f(x["dout"], ad)
            g = [torch.empty_like(t) for t in (q, k, v, lr, mom, decay, W0, W0)]
            wsb = E.workspace(shape, True, dev)

        mm, Mo = (None, None) if nomom else (mom, Me)

        def step(st=stream):
            E.e2ttt_chunk_scan_fwd(shape, q, k, v, lr, mm, decay, W0, None, outb, We, Mo, saved, ws,
                                   stream=st)
            if train:
                E.e2ttt_chunk_scan_bwd(shape, q, k, v, lr, mom, decay, saved, dout, None, None, *g,
                                       wsb, stream=st)

        for _ in range(3):
            step()
        graph = capture_graph(torch, dev, stream, step) if args.graph else None
        run = graph.replay if graph is not None else step
        for _ in range(3):
            run()
        ms = _timed(torch, stream, run, steps)
        del graph
        flops = train_flops(w) if train else fwd_flops(w)
        out[("fwd_bwd_" if train else "fwd_") + name + ("_chunk_mean" if coef else "") +
            ("_no_momentum" if nomom else "")] = {
            "value": w.B * w.T / (ms / 1e3), "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "tflops": flops / (ms / 1e3) / 1e12, "frac_bf16_peak": flops / (ms / 1e3) / 1e12 / measured_peaks()["bf16_tflops"]}
        del q, k, v, outb, We, Me, saved, ws
        torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------- our path
def run_k1_only(args):
    """K1 alone at 2^26 token-heads (the `k1_2e26` measurement of the main
    line) as its own JSON line: --warmup launches, then --steps timed ones.
    For profiling K1 by itself; not the benchmark's contract line."""
    import torch
    import test_weight_layers_chunk_b200 as E
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    r = measure_k1_large(E, torch, dev, stream, reps=args.steps)
    print(json.dumps({"metric": "K1 token-heads/s at 2^26", "value": r["token_heads"] / (r["us_per_launch"] / 1e6),
                      "unit": "token-heads/s", "k1_2e26": r}))


def run_ours(args, w):
    import torch
    import test_weight_layers_chunk_b200 as E
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        xs = gen.generate(w)
        cpu_baseline = cpu_baselines(w, xs, args.cpu_budget)
        del xs

    x = gen.generate(w, seed=w.seed + 1000 * rank)
    ad = torch.bfloat16 if w.act == gen.BF16 else torch.float32
    f = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(dt)
    q, k, v = f(x["q"], ad), f(x["k"], ad), f(x["v"], ad)
    lr, mom, decay, W0 = f(x["lr"]), f(x["mom"]), f(x["decay"]), f(x["W0"])
    M0 = None if not np.any(x["M0"]) else f(x["M0"])   # the workload's M0 is zero
    train = args.mode == "train"
    # training: the forward keeps its per-chunk E and dH for the backward
    # (save_acts), which then does not recompute them
    shape = E.make_shape(w.B, w.H, w.T, w.C, w.d_k, w.d_v, w.d_h, w.kind, w.act, w.loss,
                         save_acts=E.SAVE_ACTS if train else E.RECOMPUTE_ACTS)
    assert E.e2ttt_fwd_uses_tensor_cores(shape) == 1
    out = torch.empty_like(v)
    W_end = torch.empty_like(W0)
    M_end = torch.empty_like(W0)
    saved = E.saved_states(shape, dev) if train else None
    ws = E.workspace(shape, False, dev)
    stream = torch.cuda.current_stream(dev)

    if train:
        dout = f(x["dout"], ad)
        grads = {n: torch.empty_like(t) for n, t in (("dq", q), ("dk", k), ("dv", v), ("dlr", lr),
                                                       ("dmom", mom), ("ddecay", decay))}
        dW0g = torch.empty_like(W0)
        dM0g = torch.empty_like(W0)
        wsb = E.workspace(shape, True, dev)

    def step(st=stream):
        E.e2ttt_chunk_scan_fwd(shape, q, k, v, lr, mom, decay, W0, M0, out, W_end, M_end, saved, ws,
                               stream=st)
        if train:
            E.e2ttt_chunk_scan_bwd(shape, q, k, v, lr, mom, decay, saved, dout, None, None,
                                   grads["dq"], grads["dk"], grads["dv"], grads["dlr"],
                                   grads["dmom"], grads["ddecay"], dW0g, dM0g, wsb, stream=st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    E.e2ttt_workspace_status(ws, stream=stream)
    # The timed step replays a CUDA graph of the same C-ABI calls (all kernels,
    # copies and memsets of one step); --graph 0 times plain stream launches.
    graph = capture_graph(torch, dev, stream, step) if args.graph else None
    run_step = graph.replay if graph is not None else step
    for _ in range(3):
        run_step()
    torch.cuda.synchronize(dev)

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            run_step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    ms_max = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    # the same step with plain stream launches, for reference
    stream_ms = _timed(torch, stream, step, max(1, min(args.steps, 50))) if graph is not None else None
    # Per-kernel durations: a second timed pass of the same step with a CUDA event
    # pair around every launch on the launching stream (kept out of the first pass,
    # whose step time the events would inflate).
    tsteps = max(1, min(args.steps, 50))
    E.e2ttt_trace_enable(True)
    ev0.record(stream)
    for _ in range(tsteps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    trace = E.e2ttt_trace_summary()
    E.e2ttt_trace_enable(False)
    ms = ev0.elapsed_time(ev1)   # the traced pass: denominators of the kernel shares
    E.e2ttt_workspace_status(ws, stream=stream)
    tokens = w.B * w.T * args.steps * world
    value = tokens / (ms_max / 1e3)

    # roofline of the dominant kernel, from its algorithmic work
    peaks = measured_peaks()
    clocks = clk.summary()
    kern = trace["kernels"]
    work = kernel_work(w, M0 is not None)
    if w.kind == gen.SWIGLU and w.d_k == w.d_v:
        dd = w.d_k * w.d_h * w.B * w.H * w.C
        for n, f in BWD_SIMT_FLOPS.items():
            work[n] = ("alu", f * dd, None)
    dom = max((n for n in kern if n in work), key=lambda n: kern[n]["total_ms"])
    avg_ms = kern[dom]["total_ms"] / kern[dom]["launches"]
    if isinstance(work[dom][0], str):      # CUDA-core backward kernel: fp32 FMA bound
        flops_launch = work[dom][1]
        achieved = flops_launch / (avg_ms / 1e3) / 1e12
        peak = fp32_fma_peak_tflops(clocks.get("sm_max_mhz") or 1965.0)
        roofline = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "algorithmic_per_launch": flops_launch,
                    "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 x max SM clock"}
    else:
        flops_launch, alg_launch, impl_launch = work[dom]
        roofline = roofline_of(flops_launch, alg_launch, avg_ms / 1e3, peaks)
        roofline["implementation_bytes_per_launch"] = impl_launch
        roofline["algorithmic_bytes_per_launch"] = alg_launch
    roofline.update({"kernel": dom, "avg_launch_us": avg_ms * 1e3,
                     "traffic": recorded_traffic(dom, w.name),
                     "share_of_step": kern[dom]["total_ms"] / ms})
    step_flops = train_flops(w) if train else fwd_flops(w)
    impl_step = sum(kv["launches"] * work[n][2] for n, kv in kern.items()
                    if n in work and work[n][2] is not None) / tsteps
    alg_step = algorithmic_bytes(w)
    whole = {"achieved_tflops": step_flops / (ms_max / args.steps / 1e3) / 1e12,
             "traced_ms_per_step": ms / tsteps, "traced_steps": tsteps,
             "timed_as": "cuda_graph_replay" if graph is not None else "stream_launches",
             "stream_launch_ms_per_step": stream_ms,
             "algorithmic_bytes_per_step": alg_step,
             "implementation_bytes_per_step": impl_step,
             "implementation_over_algorithmic": impl_step / alg_step}
    whole["frac"] = whole["achieved_tflops"] / peaks["bf16_tflops"]
    if peaks.get("bf16_tflops_sustained"):
        whole["frac_sustained"] = whole["achieved_tflops"] / peaks["bf16_tflops_sustained"]
    kernels = {}
    for n, kv in kern.items():
        avg_s = kv["total_ms"] / kv["launches"] / 1e3
        kernels[n] = {"launches": kv["launches"], "avg_us": avg_s * 1e6, "share": kv["total_ms"] / ms}
        if n in work and not isinstance(work[n][0], str):
            f, alg, impl = work[n]
            r = roofline_of(f, alg, avg_s, peaks)
            kernels[n].update({"bound": r["bound"], "frac": r["frac"], "tflops": f / avg_s / 1e12,
                               "alg_gbs": alg / avg_s / 1e9, "impl_gbs": impl / avg_s / 1e9,
                               "impl_frac_hbm": impl / avg_s / 1e9 / peaks["hbm_gbs"]})

    extras = {}
    if args.extras and rank == 0 and world == 1 and not train:
        extras = measure_extras(E, torch, dev, stream, args)
    k1_large = None
    if rank == 0 and not train:
        try:   # an auxiliary measurement: its failure is reported, the line still prints
            k1_large = measure_k1_large(E, torch, dev, stream)
        except Exception as exc:  # noqa: BLE001
            k1_large = {"error": f"{type(exc).__name__}: {exc}"}

    # End to end through the public API with pinned host buffers, pipelined the way
    # a serving loop runs: every step copies its inputs in (one copy stream),
    # computes (the launching stream) and copies its results out (another copy
    # stream), on two sets of device buffers, so step i's input copies overlap
    # step i-1's compute and step i-2's output copies (the two copy directions
    # use separate copy engines). Events order each set's reuse; the timed
    # region runs from before the first input copy to after the last output copy.
    e2e = None
    if args.e2e_steps > 0:
        ins = (q, k, v, lr, mom, decay, W0)
        outs = (out, W_end, M_end)
        host_in = [t.cpu().pin_memory() for t in ins]
        dev_in = [list(ins), [t.clone() for t in ins]]
        dev_out = [list(outs), [torch.empty_like(t) for t in outs]]
        host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
                    for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = sum(t.numel() * t.element_size() for t in host_out[0])
        # input copies split over two streams (two copy engines), by size
        s_in, s_in2, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        order = sorted(range(len(ins)), key=lambda j: -host_in[j].numel() * host_in[j].element_size())
        lanes = ([], [])
        load = [0, 0]
        for j in order:   # greedy: the larger copies alternate between the two streams
            lane = 0 if load[0] <= load[1] else 1
            lanes[lane].append(j)
            load[lane] += host_in[j].numel() * host_in[j].element_size()
        ev_in = [torch.cuda.Event() for _ in range(2)]     # set b's inputs are on the device
        ev_in2 = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]   # the step on set b has finished
        ev_out = [torch.cuda.Event() for _ in range(2)]    # set b's results are on the host
        for b in range(2):
            ev_done[b].record(stream)
            ev_out[b].record(stream)

        def run_set(b):
            qi, ki, vi, lri, mi, di, Wi = dev_in[b]
            oo, We, Me = dev_out[b]
            E.e2ttt_chunk_scan_fwd(shape, qi, ki, vi, lri, mi, di, Wi, M0, oo, We, Me, saved, ws,
                                   stream=stream)
            if train:
                E.e2ttt_chunk_scan_bwd(shape, qi, ki, vi, lri, mi, di, saved, dout, None, None,
                                       grads["dq"], grads["dk"], grads["dv"], grads["dlr"],
                                       grads["dmom"], grads["ddecay"], dW0g, dM0g, wsb,
                                       stream=stream)

        def e2e_step(i):
            b = i & 1
            for st_, ev_, lane in ((s_in, ev_in, lanes[0]), (s_in2, ev_in2, lanes[1])):
                st_.wait_event(ev_done[b])     # the step two back no longer reads set b
                with torch.cuda.stream(st_):
                    for j in lane:
                        dev_in[b][j].copy_(host_in[j], non_blocking=True)
                ev_[b].record(st_)
                stream.wait_event(ev_[b])
            stream.wait_event(ev_out[b])       # set b's previous results have left
            run_set(b)
            ev_done[b].record(stream)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                for dst, src in zip(host_out[b], dev_out[b]):
                    dst.copy_(src, non_blocking=True)
            ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        s_in.wait_stream(stream)               # the first input copies start after ev0
        s_in2.wait_stream(stream)
        for i in range(args.e2e_steps):
            e2e_step(2 + i)
        stream.wait_stream(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_in2)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
        e2e = {"value": w.B * w.T * args.e2e_steps * world / (e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "pipeline": "input copies (two streams), compute and result copies of "
                           "successive steps overlapped, two device buffer sets"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if w.act == gen.BF16 else "f32",
                "data": "synthetic (seeded numpy; shapes and distributions of the workload)",
                "config": config_dict(w, argparse.Namespace(gpus=world, mode=args.mode)),
                "roofline": roofline, "step_roofline": whole, "kernels": kernels,
                "gpu_launches": trace["launches"] // tsteps * args.steps, "clocks": clocks,
                "cpu_baseline": cpu_baseline, "e2e": e2e, "k1_2e26": k1_large, "extra": extras}
        print(json.dumps(line))
    del graph, run_step  # release the captured graph before the process group
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, choices=[w.name for w in gen.WORKLOADS],
                    help="default: layer_1p3b_2k (fwd) or train_1p3b_2k (train)")
    ap.add_argument("--mode", choices=["fwd", "train", "k1"], default="fwd",
                    help="k1: only K1 at 2^26 token-heads (for profiling it alone)")
    ap.add_argument("--e2e-steps", type=int, default=30,
                    help="timed steps of the end-to-end loop; the first step's input copies and "
                         "the last one's result copies overlap nothing, so more steps measure the "
                         "steady state")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extras", type=int, default=1, help="also time T=16K fwd and T=2K fwd+bwd")
    ap.add_argument("--extra-steps", type=int, default=20)
    ap.add_argument("--graph", type=int, default=1,
                    help="time replays of a CUDA graph of the step (0: plain stream launches)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload is None:
        args.workload = "train_1p3b_2k" if args.mode == "train" else "layer_1p3b_2k"
    w = gen.BY_NAME[args.workload]
    if args.mode == "k1":
        run_k1_only(args)
    elif args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
