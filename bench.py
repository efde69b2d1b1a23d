"""Benchmark of the BATQuant W4A4 linear hot path on B200.

One step = one pass of the whole path over one batch of the largest single-GPU workload: the
seven linears of one Qwen3-8B-shaped decoder layer at S = 8192 tokens (q 4096->4096, k and v
4096->1024, o 4096->4096, gate and up 4096->12288, down 12288->4096), each with its own seeded
bf16 activations, transform, clip logits and prepared weights, each through batq_linear
(batq_quant_act: GPK transform + clip + MXFP4 into the tcgen05 scale layout, then
batq_gemm_mxfp4: block-scaled tensor-core GEMM, fp32 out).  The weights are prepared offline
(untimed), as in the method.

Prints one JSON line.  ``value`` is the step's GEMM-equivalent throughput (2*S*N*M flops of the
seven linears per step / device step time, summed over ranks).  ``roofline`` is the dominant
kernel's (the pair GEMM) against the dense FP4 peak; ``roofline_quant`` the quantiser's against
HBM.  ``per_config`` holds the other workloads (q_proj and down_proj prefill, decode, the W4A8,
NVFP4, naive-Kronecker, KV-cache and RMSNorm rows).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl batq|reference]
    python bench.py --only quant|gemm|linear --workload NAME [--launches n]   (one kernel, for ncu)

Multi-GPU (torchrun): every rank runs its own batch (weak scaling, no data-path collective);
times are the max over ranks.  ``--impl reference`` times the CPU oracle on a bounded sample of
the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BAT+clip+MXFP4 quant GB/s & W4A4 GEMM TFLOPS (% of HBM / FP4 roofline)"
WORKLOAD = ("Qwen3-8B-shaped decoder layer, 7 linears at S=8192 (q,k,v,o,gate,up,down; "
            "N->M 4096->4096/1024/1024/4096/12288/12288, 12288->4096), bf16 X, W4A4 MXFP4, fp32 out")
QUANT_BYTES_PER_ELEM = 2 + 0.5 + 1.0 / 32  # bf16 in, E2M1 codes + E8M0 scales out
FP4_NOMINAL_OVER_BF16 = 9.0 / 2.25         # dense fp4 / dense bf16 nominal ratio
REPEATS = 5                                # every per-kernel loop: median of this many repeats
CSRC = os.path.join(ROOT, "mxfp4_w4a4_post_block_b200", "csrc")

# DRAM bytes (read + write) of one layer step's launch of each grouped kernel, from an ncu capture of
# `bench.py --only group --workload layer` (metrics dram__bytes_read.sum, dram__bytes_write.sum),
# valid only for the kernel sources whose hash is recorded with it: a changed kernel reports null.
NCU_TRAFFIC = {
    "k_gemm_pair": {"src": "a496fbeb3db1df9c", "bytes_per_step": 374014208 + 1235212032},
    "k_quant_act_tc": {"src": "e53a61cae13ec272", "bytes_per_step": 605399040 + 143117056},
}
TRAFFIC_SOURCES = {
    "k_gemm_pair": ("gemm_pair.cu", "ptx.cuh", "kernels.h", "host_util.h", "host_util.cpp"),
    "k_quant_act_tc": ("quant_act_tc.cu", "quant_act.cu", "quant_common.cuh", "ptx.cuh", "kernels.h",
                       "host_util.h", "host_util.cpp"),
}


def _code_only(text):
    """Source text without C/C++ comments and whitespace runs, so that a comment edit does not mark a
    recorded capture stale (the compiled kernel is the same)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_hash(kernel):
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, launches_per_step):
    """Per-launch DRAM traffic of `kernel` from the recorded capture, or None if it is stale."""
    rec = NCU_TRAFFIC[kernel]
    if rec["bytes_per_step"] is None or rec["src"] != source_hash(kernel):
        return None
    return rec["bytes_per_step"] / launches_per_step


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML during the timed region."""

    def __init__(self, device_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self._h = None
            self.error = repr(e)

    def _run(self):
        nv = self._nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_power_brake": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while True:
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for n, bit in names.items():
                    if r & bit:
                        self.reasons.add(n)
            except Exception:  # noqa: BLE001
                pass
            if self._stop.wait(0.002):
                break

    def __enter__(self):
        if self._h is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(values, device=None):
    """Each value's maximum over all ranks (unchanged with one rank): a multi-GPU time is the
    slowest rank's.  Every rank must call this the same number of times."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_tflops(world_size, flops_per_rank_step, ms_per_step):
    """Whole-job throughput: every rank processes its own batch of flops_per_rank_step in the
    (max-over-ranks) step time (weak scaling)."""
    return world_size * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def _cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


# ------------------------------------------------------------------ CPU oracle legs

def _oracle_layer(workloads=None):
    """The seven layer workloads (drawn here unless given) and their oracle-prepared weights
    (offline, untimed)."""
    from mxfp4_w4a4_post_block_b200 import workloads as WL
    from oracle import batq_oracle as O
    if workloads is None:
        workloads = [WL.layer_linear(j) for j in range(len(WL.LAYER_LINEARS))]
    out = []
    for w in workloads:
        wp = O.prepare_weights(w.W, w.A, w.B)
        out.append((w, {"codes": wp["codes"], "scales": wp["scales"]}))
        w.W = None
    return out


def _oracle_rows(w, wp, rows):
    """One linear of the step on `rows` tokens: quant_act, then the fp64 GEMM against every
    prepared weight row."""
    from oracle import batq_oracle as O
    act = O.quant_act(w.x[rows], w.A, w.B, w.alpha_min, w.alpha_max)
    out, _ = O.gemm(act["codes"], act["scales"], wp["codes"], wp["scales"])
    return out


def cpu_baseline(layer, rows_per_linear=128):
    """The oracle timed on this host over a bounded sample of one layer step: the same number of
    tokens of each of the seven linears through quant_act and the fp64 GEMM against all of that
    linear's prepared weight rows."""
    _oracle_rows(layer[1][0], layer[1][1], np.arange(8))  # first-call overheads stay out
    flops, t = 0.0, 0.0
    for j, (w, wp) in enumerate(layer):
        rows = np.arange(rows_per_linear) + j * 97 % (w.S - rows_per_linear)
        t0 = time.perf_counter()
        _oracle_rows(w, wp, rows)
        t += time.perf_counter() - t0
        flops += 2.0 * len(rows) * w.N * w.M
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": _cpu_cores(), "kind": "oracle",
            "sample": f"{rows_per_linear} of the 8192 tokens of each of the 7 linears of the layer step "
                      f"(quant_act + fp64 GEMM against all prepared weight rows), {t:.2f} s"}


def run_reference(args):
    """The oracle as the reference arm: each step is a bounded sample of the layer step (rows of
    one linear, cycling through the seven), timed on the host cores."""
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    layer = _oracle_layer()
    _oracle_rows(layer[1][0], layer[1][1], np.arange(8))
    t0 = time.perf_counter()
    _oracle_rows(layer[0][0], layer[0][1], np.arange(32))
    t_probe = time.perf_counter() - t0
    budget = 150.0 / (args.steps + args.warmup)  # seconds per step
    rows = int(max(8, min(1024, 32 * budget / max(t_probe, 1e-3))))
    for i in range(args.warmup):
        w, wp = layer[i % 7]
        _oracle_rows(w, wp, np.arange(rows))
    flops, t = 0.0, 0.0
    for i in range(args.steps):
        w, wp = layer[i % 7]
        r0 = (i * rows) % (w.S - rows)
        t1 = time.perf_counter()
        _oracle_rows(w, wp, np.arange(r0, r0 + rows))
        t += time.perf_counter() - t1
        flops += 2.0 * rows * w.N * w.M
    value = flops / t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": layer_config(1),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _cpu_cores(), "kind": "oracle",
                             "sample": f"{rows} tokens of one linear per step (cycling q,k,v,o,gate,up,down), "
                                       f"quant_act + fp64 GEMM against all of its prepared weight rows"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ device workloads

def layer_config(ws):
    return {"workload": WORKLOAD, "S": 8192, "linears": "q,k,v,o,gate,up,down",
            "l2": "inputs larger than L2: one step reads 604 MB of activations and 102 MB of prepared weights "
                  "and writes 1.27 GB of fp32 output",
            "parallelism": f"replicas x{ws} (independent batches)"}


def _bf16(w, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(w.x_bits).view(np.int16)).view(torch.bfloat16).to(dev)


def linear_set(w, dev, real_weights=True, out_dtype=None, gen=None):
    """Device buffers of one linear: X, B, ratios, prepared weights, workspace (codes and MMA
    scales), output.  With real_weights the weights are W prepared by batq_prepare_weights;
    otherwise random codes with unit scales (timing does not depend on their values)."""
    import torch

    from mxfp4_w4a4_post_block_b200 import batq as BQ
    S, N, M = w.S, w.N, w.M
    z = {"w": w, "S": S, "N": N, "M": M, "A": w.A, "X": _bf16(w, dev),
         "B": torch.from_numpy(np.ascontiguousarray(w.B.reshape(-1))).to(dev),
         "ratios": torch.from_numpy(BQ.batq_clip_ratios(w.alpha_min, w.alpha_max)).to(dev)}
    wc, wsc = BQ.empty_act_buffers(M, N, device=dev)
    if real_weights:
        Wd = torch.from_numpy(w.W).to(dev)
        pws = torch.empty(BQ.batq_prepare_workspace_size(N), dtype=torch.uint8, device=dev)
        BQ.batq_prepare_weights(Wd, w.A, w.B, wc, wsc, pws)
        del Wd, pws
    else:
        wc.random_(0, 256, generator=gen)
        wsc.fill_(127)
    z["wc"], z["wsc"] = wc, wsc
    lws = torch.empty(BQ.batq_linear_workspace_size(S, N), dtype=torch.uint8, device=dev)
    code_bytes = -(-S * (N // 2) // 256) * 256
    z["lws"], z["codes"], z["scales"] = lws, lws[:S * (N // 2)].view(S, N // 2), lws[code_bytes:]
    z["out"] = torch.empty((S, M), dtype=out_dtype or torch.float32, device=dev)
    return z


def launcher(kind, z, sp):
    """A closure launching one kernel (or the whole linear) of set z on stream sp."""
    from mxfp4_w4a4_post_block_b200 import batq as BQ
    if kind == "linear":
        return lambda: BQ.batq_linear(z["X"], z["A"], z["B"], z["ratios"], z["wc"], z["wsc"], z["M"], z["lws"],
                                      z["out"], stream=sp)
    if kind == "quant":
        return lambda: BQ.batq_quant_act(z["X"], z["A"], z["B"], z["ratios"], z["codes"], z["scales"],
                                         BQ.BATQ_SCALES_MMA, stream=sp)
    if kind == "gemm":
        return lambda: BQ.batq_gemm_mxfp4(z["codes"], z["scales"], z["wc"], z["wsc"], z["S"], z["M"], z["N"],
                                          z["out"], stream=sp)
    raise ValueError(kind)


class Timer:
    """CUDA-event timing on the launching stream; counts the library launches it times."""

    def __init__(self, stream):
        self.stream = stream
        self.launches = 0

    def once(self, fns, reps=1, kernels_per_fn=1):
        """ms per pass over fns (reps passes back to back between two events)."""
        import torch
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for _ in range(reps):
            for f in fns:
                f()
        e1.record(self.stream)
        torch.cuda.synchronize()
        self.launches += reps * len(fns) * kernels_per_fn
        return e0.elapsed_time(e1) / reps

    def median(self, fns, reps=1, kernels_per_fn=1, repeats=REPEATS):
        """Median over `repeats` of once()."""
        for f in fns:
            f()
        return statistics.median(self.once(fns, reps, kernels_per_fn) for _ in range(repeats))

    def each(self, fns, repeats=REPEATS):
        """ms of each of fns within one back-to-back pass over all of them (events between the
        launches), median over `repeats` passes."""
        import torch
        for f in fns:
            f()
        per = [[] for _ in fns]
        for _ in range(repeats):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
            ev[0].record(self.stream)
            for i, f in enumerate(fns):
                f()
                ev[i + 1].record(self.stream)
            torch.cuda.synchronize()
            for i in range(len(fns)):
                per[i].append(ev[i].elapsed_time(ev[i + 1]))
            self.launches += len(fns)
        return [statistics.median(p) for p in per]


def per_config(dev, peaks, timer, sp):
    """The other workloads, each timed as the median of five repeats of back-to-back launches whose
    inputs rotate through more than the 126 MB L2."""
    import torch

    from mxfp4_w4a4_post_block_b200 import batq as BQ
    from mxfp4_w4a4_post_block_b200 import workloads as WL

    fp4_peak = peaks["bf16_tflops"] * FP4_NOMINAL_OVER_BF16
    hbm = peaks["hbm_gbs"]
    res = {}

    def prefill(name, w, copies, reps):
        sets = [linear_set(w, dev, real_weights=(c == 0)) for c in range(copies)]
        for z in sets[1:]:
            z["wc"].copy_(sets[0]["wc"])
            z["wsc"].copy_(sets[0]["wsc"])
        S, N, M = w.S, w.N, w.M
        l_ms = timer.median([launcher("linear", z, sp) for z in sets], reps, 2) / copies
        q_ms = timer.median([launcher("quant", z, sp) for z in sets], reps) / copies
        g_ms = timer.median([launcher("gemm", z, sp) for z in sets], reps) / copies
        qb, fl = S * N * QUANT_BYTES_PER_ELEM, 2.0 * S * N * M
        res[name] = {"linear_us": l_ms * 1e3, "linear_tflops": fl / l_ms / 1e9,
                     "quant_us": q_ms * 1e3, "quant_gbs": qb / q_ms / 1e6, "quant_frac_hbm": qb / q_ms / 1e6 / hbm,
                     "gemm_us": g_ms * 1e3, "gemm_tflops": fl / g_ms / 1e9, "gemm_frac_fp4": fl / g_ms / 1e9 / fp4_peak}
        del sets

    # q_proj prefill (S=2048): ten sets of 64 MB rotate through the L2
    prefill("q_proj_2048x4096x4096", WL.q_proj(), 10, 3)
    # down_proj prefill (S=4096, N=12288): three sets of 250 MB
    prefill("down_proj_4096x12288x4096", WL.down_proj(), 3, 2)

    # decode: S in {1, 4, 16}, N=4096, M=24576; the GEMM streams 53.5 MB of prepared weights
    g = torch.Generator(device=dev).manual_seed(4)
    for S in (1, 4, 16):
        w = WL.decode(S, with_w=False)
        sets = [linear_set(w, dev, real_weights=False, gen=g) for _ in range(3)]
        q_ms = timer.median([launcher("quant", z, sp) for z in sets], 10) / 3
        g_ms = timer.median([launcher("gemm", z, sp) for z in sets], 10) / 3
        l_ms = timer.median([launcher("linear", z, sp) for z in sets], 10, 2) / 3
        wb = w.M * w.N * (0.5 + 1.0 / 32)
        res[f"decode_{S}x4096x24576"] = {
            "quant_us": q_ms * 1e3, "gemm_us": g_ms * 1e3, "gemm_weight_gbs": wb / g_ms / 1e6,
            "gemm_frac_hbm": wb / g_ms / 1e6 / hbm, "linear_us": l_ms * 1e3, "linear_weight_gbs": wb / l_ms / 1e6}
        del sets
    res["decode_note"] = ("launch-bound quantiser; GEMM judged on weight bytes against HBM; linear = batq_linear "
                          "(the GEMM prefetches its weights into L2 while the quantiser runs)")

    # a decode step of the layer's seven linears at S = 16 (102 MB of prepared weights): one
    # batq_linear_grouped call (one quantiser launch, one single-CTA GEMM launch) against seven
    # batq_linear calls; two sets rotate (204 MB of weights, more than L2)
    dsets = [[linear_set(WL.layer_linear(j, S=16, with_w=False), dev, real_weights=False, gen=g)
              for j in range(len(WL.LAYER_LINEARS))] for _ in range(2)]
    dwb = sum(z["M"] * z["N"] * (0.5 + 1.0 / 32) for z in dsets[0])
    dgroups = []
    for zs in dsets:
        gl = [dict(X=z["X"], A=z["A"], B=z["B"], ratios=z["ratios"], w_codes=z["wc"], w_scales=z["wsc"],
                   M=z["M"], out=z["out"]) for z in zs]
        gws = torch.empty(BQ.batq_linear_grouped_workspace_size([(z["S"], z["N"]) for z in zs]),
                          dtype=torch.uint8, device=dev)
        dgroups.append(BQ.prepare_linear_grouped(gl, gws))  # marshalled once: one ctypes call per step
    grp_ms = timer.median([lambda f=f: f(sp) for f in dgroups], 10, 2) / 2
    per_ms = timer.median([launcher("linear", z, sp) for zs in dsets for z in zs], 10, 2) / 2
    res["decode_layer_16x7_linears"] = {
        "grouped_us": grp_ms * 1e3, "grouped_weight_gbs": dwb / grp_ms / 1e6,
        "grouped_frac_hbm": dwb / grp_ms / 1e6 / hbm, "per_linear_calls_us": per_ms * 1e3,
        "per_linear_weight_gbs": dwb / per_ms / 1e6,
        "note": "q, k, v, o, gate, up, down at 16 tokens; batq_linear_grouped vs seven batq_linear calls"}
    del dsets, dgroups

    w = WL.q_proj(with_w=False)
    S, N, M = w.S, w.N, w.M
    X = _bf16(w, dev)
    B = torch.from_numpy(np.ascontiguousarray(w.B.reshape(-1))).to(dev)
    r = torch.from_numpy(BQ.batq_clip_ratios(w.alpha_min, w.alpha_max)).to(dev)
    fl = 2.0 * S * N * M

    # W4A8 on q_proj: MXFP8 activations (3.03 B per element moved), E4M3 x E4M3 GEMM (FP8 peak =
    # measured bf16 x 2)
    g8 = torch.Generator(device=dev).manual_seed(7)
    sets = []
    for c in range(6):
        codes8, sc8 = BQ.empty_mxfp8_buffers(S, N, device=dev)
        wc8 = torch.empty((M, N), dtype=torch.uint8, device=dev).random_(0, 128, generator=g8)
        wc8[(wc8 & 0x7F) == 0x7F] = 0x38  # no NaN codes
        _, wsb = BQ.batq_mxfp8_buffer_sizes(M, N)
        sets.append({"X": X if c == 0 else X.clone(), "codes": codes8, "scales": sc8, "wc": wc8,
                     "wsc": torch.full((wsb,), 127, dtype=torch.uint8, device=dev),
                     "out": torch.empty((S, M), dtype=torch.float32, device=dev)})
    q_ms = timer.median([lambda z=z: BQ.batq_quant_act_mxfp8(z["X"], w.A, B, r, z["codes"], z["scales"], stream=sp)
                         for z in sets], 3) / 6
    g_ms = timer.median([lambda z=z: BQ.batq_gemm_w4a8(z["codes"], z["scales"], z["wc"], z["wsc"], S, M, N, z["out"],
                                                       stream=sp) for z in sets], 3) / 6
    qb = S * N * (2 + 1 + 1.0 / 32)
    res["w4a8_q_proj_2048x4096x4096"] = {
        "quant_us": q_ms * 1e3, "quant_gbs": qb / q_ms / 1e6, "quant_frac_hbm": qb / q_ms / 1e6 / hbm,
        "gemm_us": g_ms * 1e3, "gemm_tflops": fl / g_ms / 1e9, "gemm_frac_fp8": fl / g_ms / 1e9 / (2 * peaks["bf16_tflops"]),
        "note": "MXFP8 activations x MXFP4 weights in E4M3 containers (kind::mxf8f6f4); FP8 peak = measured bf16 x 2"}
    del sets

    # NVFP4 output on q_proj (E4M3 scale per 16, per-tensor encode scale 2.0; kind::mxf4nvf4)
    gsn = torch.full((1,), 2.0, dtype=torch.float32, device=dev)
    gn = torch.Generator(device=dev).manual_seed(11)
    sets = []
    for c in range(6):
        cn, sn = BQ.empty_nvfp4_buffers(S, N, device=dev)
        wcn, wsn = BQ.empty_nvfp4_buffers(M, N, device=dev)
        wcn.random_(0, 256, generator=gn)
        wsn.fill_(0x38)  # E4M3 1.0
        sets.append({"X": X if c == 0 else X.clone(), "codes": cn, "scales": sn, "wc": wcn, "wsc": wsn,
                     "out": torch.empty((S, M), dtype=torch.float32, device=dev)})
    q_ms = timer.median([lambda z=z: BQ.batq_quant_act_nvfp4(z["X"], w.A, B, r, z["codes"], z["scales"], gs=gsn,
                                                             stream=sp) for z in sets], 3) / 6
    g_ms = timer.median([lambda z=z: BQ.batq_gemm_nvfp4(z["codes"], z["scales"], gsn, z["wc"], z["wsc"], None, S, M,
                                                        N, z["out"], stream=sp) for z in sets], 3) / 6
    qb = S * N * (2 + 0.5 + 1.0 / 16)
    res["nvfp4_q_proj_2048x4096x4096"] = {
        "quant_us": q_ms * 1e3, "quant_gbs": qb / q_ms / 1e6, "quant_frac_hbm": qb / q_ms / 1e6 / hbm,
        "gemm_us": g_ms * 1e3, "gemm_tflops": fl / g_ms / 1e9, "gemm_frac_fp4": fl / g_ms / 1e9 / fp4_peak}
    del sets

    # naive Kronecker (one A_i per block) on q_proj: quantiser and whole linear
    wk = WL.with_naive_kronecker(WL.q_proj(), seed=9)
    Ak = torch.from_numpy(np.ascontiguousarray(wk.A.reshape(-1))).to(dev)
    sets = []
    for c in range(8):
        wc, wsc = BQ.empty_act_buffers(M, N, device=dev)
        if c == 0:
            Wd = torch.from_numpy(wk.W).to(dev)
            pws = torch.empty(BQ.batq_prepare_weights_kron_workspace_size(N), dtype=torch.uint8, device=dev)
            BQ.batq_prepare_weights_kron(Wd, wk.A, wk.B, wc, wsc, pws)
            del Wd, pws
        else:
            wc.copy_(sets[0]["wc"])
            wsc.copy_(sets[0]["wsc"])
        codes, scales = BQ.empty_act_buffers(S, N, device=dev)
        sets.append({"X": X if c == 0 else X.clone(), "codes": codes, "scales": scales, "wc": wc, "wsc": wsc,
                     "lws": torch.empty(BQ.batq_linear_workspace_size(S, N), dtype=torch.uint8, device=dev),
                     "out": torch.empty((S, M), dtype=torch.float32, device=dev)})
    q_ms = timer.median([lambda z=z: BQ.batq_quant_act_kron(z["X"], Ak, B, r, z["codes"], z["scales"], stream=sp)
                         for z in sets], 3) / 8
    l_ms = timer.median([lambda z=z: BQ.batq_linear_kron(z["X"], Ak, B, r, z["wc"], z["wsc"], M, z["lws"], z["out"],
                                                         stream=sp) for z in sets], 3, 2) / 8
    qb = S * N * QUANT_BYTES_PER_ELEM
    res["naive_kron_q_proj_2048x4096x4096"] = {
        "quant_us": q_ms * 1e3, "quant_gbs": qb / q_ms / 1e6, "quant_frac_hbm": qb / q_ms / 1e6 / hbm,
        "linear_us": l_ms * 1e3, "linear_tflops": fl / l_ms / 1e9,
        "note": "P_i = B_i (x) A_i with one 8x8 A_i per block (10,240 parameters at N=4096); the quantiser reads "
                "256 B of A_i per block column and tile on top of the GPK bytes"}
    del sets

    # BAT on the KV cache: 8192 new tokens of one layer's K (8 KV heads x 128 = 1024 elements per
    # token) written into a paged cache of 16384 slots through a permuted slot mapping; eight sets
    # rotate through the L2
    Skv, Nkv = 8192, 1024
    wkv = WL.custom(Skv, Nkv, 16, 33, with_w=False)
    Xkv = _bf16(wkv, dev)
    Bkv = torch.from_numpy(np.ascontiguousarray(wkv.B.reshape(-1))).to(dev)
    rkv = torch.from_numpy(BQ.batq_clip_ratios(wkv.alpha_min, wkv.alpha_max)).to(dev)
    slots = torch.randperm(2 * Skv, generator=torch.Generator().manual_seed(5))[:Skv].to(torch.int32).to(dev)
    for fmt, name, cb in ((BQ.BATQ_KV_MXFP4, "kv4", 0.5), (BQ.BATQ_KV_MXFP8, "kv8", 1.0)):
        sets = []
        for c in range(8):
            cc = torch.zeros((2 * Skv, int(Nkv * cb)), dtype=torch.uint8, device=dev)
            cs = torch.zeros((2 * Skv, Nkv // 32), dtype=torch.uint8, device=dev)
            sets.append((Xkv if c == 0 else Xkv.clone(), cc, cs))
        q_ms = timer.median([lambda s=s, fmt=fmt: BQ.batq_quant_kv_cache(s[0], wkv.A, Bkv, rkv, slots, s[1], s[2],
                                                                         kv_format=fmt, stream=sp)
                             for s in sets], 3) / 8
        qb = Skv * Nkv * (2 + cb + 1.0 / 32) + Skv * 4
        res[f"kv_cache_{name}_{Skv}x{Nkv}"] = {"quant_us": q_ms * 1e3, "quant_gbs": qb / q_ms / 1e6,
                                               "quant_frac_hbm": qb / q_ms / 1e6 / hbm}
        del sets
    torch.cuda.empty_cache()
    return res


def run_only(args):
    """A few launches of one kernel on one workload, for profiling (no timing, no JSON).  The weights
    are random codes with unit scales, so no weight-preparation kernel runs before them; with
    --only gemm one quantiser launch per linear first fills the activation codes."""
    import torch

    from mxfp4_w4a4_post_block_b200 import batq as BQ
    from mxfp4_w4a4_post_block_b200 import workloads as WL
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    names = [n for n, _, _ in WL.LAYER_LINEARS]
    if args.workload == "layer":
        ws = [WL.layer_linear(j) for j in range(len(names))]
    elif args.workload.startswith("layer_"):
        ws = [WL.layer_linear(names.index(args.workload[6:]))]
    elif args.workload == "q_proj":
        ws = [WL.q_proj()]
    elif args.workload == "down_proj":
        ws = [WL.down_proj()]
    elif args.workload.startswith("decode"):
        ws = [WL.decode(int(args.workload[6:]))]
    else:
        raise SystemExit(f"unknown workload {args.workload}")
    g = torch.Generator(device=dev).manual_seed(1)
    sets = [linear_set(w, dev, real_weights=False, gen=g) for w in ws]
    sp = torch.cuda.current_stream(dev).cuda_stream
    if args.only == "gemm":
        for z in sets:
            launcher("quant", z, sp)()
    torch.cuda.synchronize()
    if args.only == "group":
        group = [dict(X=z["X"], A=z["A"], B=z["B"], ratios=z["ratios"], w_codes=z["wc"], w_scales=z["wsc"],
                      M=z["M"], out=z["out"]) for z in sets]
        gws = torch.empty(BQ.batq_linear_grouped_workspace_size([(z["S"], z["N"]) for z in sets]),
                          dtype=torch.uint8, device=dev)
    for _ in range(args.launches):
        if args.only == "group":
            BQ.batq_linear_grouped(group, gws, stream=sp)
            continue
        for z in sets:
            launcher(args.only, z, sp)()
    torch.cuda.synchronize()
    if BQ.batq_device_error() != 0:
        raise SystemExit("device error word set")
    print(f"{args.only} x{args.launches} on {args.workload}: ok")
    return 0


def run_batq(args):
    import torch
    import torch.distributed as dist

    from mxfp4_w4a4_post_block_b200 import batq as BQ
    from mxfp4_w4a4_post_block_b200 import workloads as WL

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    peaks = _peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_NOMINAL_OVER_BF16

    # the layer: seven linears, each with its own inputs and prepared weights
    workloads = [WL.layer_linear(j) for j in range(len(WL.LAYER_LINEARS))]
    layer = [linear_set(w, dev) for w in workloads]
    flops = sum(2.0 * z["S"] * z["N"] * z["M"] for z in layer)
    qbytes = sum(z["S"] * z["N"] * QUANT_BYTES_PER_ELEM for z in layer)
    # One step: the seven independent linears through batq_linear_grouped (one quantiser launch over
    # all activations, one CTA-pair GEMM launch over all products).  For comparison the same step as
    # seven batq_linear calls.
    group = [dict(X=z["X"], A=z["A"], B=z["B"], ratios=z["ratios"], w_codes=z["wc"], w_scales=z["wsc"], M=z["M"],
                  out=z["out"]) for z in layer]
    gws = torch.empty(BQ.batq_linear_grouped_workspace_size([(z["S"], z["N"]) for z in layer]), dtype=torch.uint8,
                      device=dev)
    quant_group = [dict(X=z["X"], A=z["A"], B=z["B"], ratios=z["ratios"], codes=z["codes"], scales=z["scales"])
                   for z in layer]
    gemm_group = [dict(a_codes=z["codes"], a_scales=z["scales"], w_codes=z["wc"], w_scales=z["wsc"], S=z["S"],
                       M=z["M"], N=z["N"], out=z["out"]) for z in layer]
    per_linear_fns = [launcher("linear", z, sp) for z in layer]
    # the grouped calls with their arguments marshalled once (one ctypes call per launch)
    run_group = BQ.prepare_linear_grouped(group, gws)
    run_quant_group = BQ.prepare_quant_act_grouped(quant_group)
    run_gemm_group = BQ.prepare_gemm_mxfp4_grouped(gemm_group)

    def step():
        run_group(sp)

    def step_per_linear():
        for f in per_linear_fns:
            f()

    warm = max(3, args.warmup)
    for _ in range(warm):
        step()
        step_per_linear()
    torch.cuda.synchronize()
    assert BQ.batq_device_error() == 0
    timer = Timer(stream)

    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        # timed region 1: exactly K whole steps back to back (-> value)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        local_ms = e0.elapsed_time(e1) / args.steps
        # the same K steps as seven batq_linear calls each (context: what grouping saves)
        e0.record(stream)
        for _ in range(args.steps):
            step_per_linear()
        e1.record(stream)
        torch.cuda.synchronize()
        per_linear_ms = e0.elapsed_time(e1) / args.steps
        timer.launches += 2 * len(layer) * args.steps
        # timed region 2: each grouped kernel alone (one launch covers the seven linears), median of
        # five repeats of three launches back to back (-> per-kernel throughput and roofline)
        q_ms = timer.median([lambda: run_quant_group(sp)], reps=3)
        g_ms = timer.median([lambda: run_gemm_group(sp)], reps=3)
        # each linear's own kernels, one back-to-back pass with events between the launches
        q_each = timer.each([launcher("quant", z, sp) for z in layer])
        g_each = timer.each([launcher("gemm", z, sp) for z in layer])
    if ws > 1:
        dist.barrier()
    local_ms, q_ms, g_ms, per_linear_ms = max_over_ranks([local_ms, q_ms, g_ms, per_linear_ms], device=dev)
    assert BQ.batq_device_error() == 0

    # End to end through the public call with host buffers: every step uploads each linear's bf16
    # activations from pinned host memory and downloads its fp32 output.  Upload, compute and
    # download run on three streams, double-buffered across the linears.
    n_lin = len(layer)
    Xh = [z["X"].cpu().pin_memory() for z in layer]
    outh = [torch.empty(tuple(z["out"].shape), dtype=torch.float32).pin_memory() for z in layer]
    xmax = max(z["X"].numel() for z in layer)
    omax = max(z["out"].numel() for z in layer)
    Xd = [torch.empty(xmax, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    outd = [torch.empty(omax, dtype=torch.float32, device=dev) for _ in range(2)]
    s_up, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(nsteps):
        n = nsteps * n_lin
        up = [torch.cuda.Event() for _ in range(n)]
        done = [torch.cuda.Event() for _ in range(n)]
        dn = [torch.cuda.Event() for _ in range(n)]
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record(s_up)
        stream.wait_event(ea)
        s_dn.wait_event(ea)
        for i in range(n):
            z, b = layer[i % n_lin], i % 2
            S, N, M = z["S"], z["N"], z["M"]
            xd = Xd[b][:S * N].view(S, N)
            od = outd[b][:S * M].view(S, M)
            if i >= 2:
                s_up.wait_event(done[i - 2])  # Xd[b] no longer read
            with torch.cuda.stream(s_up):
                xd.copy_(Xh[i % n_lin], non_blocking=True)
            up[i].record(s_up)
            stream.wait_event(up[i])
            if i >= 2:
                stream.wait_event(dn[i - 2])  # outd[b] already downloaded
            BQ.batq_linear(xd, z["A"], z["B"], z["ratios"], z["wc"], z["wsc"], M, z["lws"], od, stream=sp)
            done[i].record(stream)
            s_dn.wait_event(done[i])
            with torch.cuda.stream(s_dn):
                outh[i % n_lin].copy_(od, non_blocking=True)
            dn[i].record(s_dn)
        s_up.wait_event(dn[n - 1])
        eb.record(s_up)
        torch.cuda.synchronize()
        return ea.elapsed_time(eb) / nsteps

    e2e_run(1)
    e2e_steps = max(2, min(args.steps, 5))
    e2e_ms = e2e_run(e2e_steps)
    (e2e_ms,) = max_over_ranks([e2e_ms], device=dev)
    del Xd, outd

    gemm_tflops = flops / (g_ms * 1e-3) / 1e12
    quant_gbs = qbytes / (q_ms * 1e-3) / 1e9
    alg_gemm_bytes = sum(z["S"] * z["N"] * (0.5 + 1 / 32) + z["M"] * z["N"] * (0.5 + 1 / 32) + z["S"] * z["M"] * 4
                         for z in layer)
    names = [n for n, _, _ in WL.LAYER_LINEARS]
    line = {
        "metric": METRIC,
        "value": whole_job_tflops(ws, flops, local_ms),
        "unit": "TFLOP/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": warm,
        "ms_per_step": local_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e2m1",
        "data": "synthetic",
        "config": layer_config(ws),
        "tokens_per_s": ws * 8192 / (local_ms * 1e-3),
        "quant_gbs": quant_gbs,
        "quant_ms": q_ms,
        "gemm_tflops": gemm_tflops,
        "gemm_ms": g_ms,
        "per_linear_calls": {"ms_per_step": per_linear_ms, "value": whole_job_tflops(ws, flops, per_linear_ms),
                             "note": "the same step as seven batq_linear calls (14 launches) instead of one "
                                     "batq_linear_grouped call (2 launches)"},
        "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": gemm_tflops / fp4_peak, "traffic": ncu_traffic("k_gemm_pair", 1),
                     "algorithmic_bytes": alg_gemm_bytes, "kernel": "k_gemm_pair",
                     "per_launch": "one grouped launch: the seven GEMMs of one step",
                     "peak_note": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} x 4 (nominal fp4/bf16)"},
        "roofline_quant": {"bound": "hbm", "achieved": quant_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": quant_gbs / peaks["hbm_gbs"], "traffic": ncu_traffic("k_quant_act_tc", 1),
                           "algorithmic_bytes": qbytes, "kernel": "k_quant_act_tc",
                           "per_launch": "one grouped launch: the seven activations of one step",
                           "peak_note": f"{peaks['source']} HBM copy"},
        "per_linear": {n: {"quant_us": q * 1e3, "quant_gbs": z["S"] * z["N"] * QUANT_BYTES_PER_ELEM / q / 1e6,
                           "gemm_us": g * 1e3, "gemm_tflops": 2.0 * z["S"] * z["N"] * z["M"] / g / 1e9}
                       for n, z, q, g in zip(names, layer, q_each, g_each)},
        "e2e": {"value": whole_job_tflops(ws, flops, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in Xh)),
                "d2h_bytes_per_step": int(sum(t.numel() * t.element_size() for t in outh)), "ms_per_step": e2e_ms,
                "note": "batq_linear on pinned host buffers for all seven linears; upload, compute and download on "
                        "three streams, double-buffered across linears"},
        "timing": "CUDA events on the launching stream; value: exactly K whole steps back to back (one "
                  "batq_linear_grouped call each); quantiser / GEMM figures and roofline: median of 5 repeats of "
                  "3 grouped launches back to back; per_linear: each linear's own kernels with events between "
                  "launches; gpu_launches counts the library launches between the two events that time value",
        "clocks": clk.summary(),
    }
    del Xh, outh
    if rank == 0 and not args.no_configs:
        line["per_config"] = per_config(dev, peaks, timer, sp)
    # library kernels launched between the two events that time `value` (one grouped quantiser and
    # one grouped GEMM per step); the other timed loops launch timer.launches more
    line["gpu_launches"] = 2 * args.steps
    line["gpu_launches_other_timed_loops"] = timer.launches
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        del layer
        torch.cuda.empty_cache()
        line["cpu_baseline"] = cpu_baseline(_oracle_layer(workloads))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description="BATQuant W4A4 linear benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["batq", "reference"], default="batq")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload kernel timings")
    ap.add_argument("--only", choices=["quant", "gemm", "linear", "group"],
                    help="launch one kernel (group: the grouped linear call) a few times (profiling)")
    ap.add_argument("--workload", default="layer", help="with --only: layer, layer_<q|k|v|o|gate|up|down>, "
                                                        "q_proj, down_proj, decode<1|4|16>")
    ap.add_argument("--launches", type=int, default=2)
    args = ap.parse_args()
    if args.only:
        return run_only(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_batq(args)


if __name__ == "__main__":
    sys.exit(main())
