"""Benchmark of the BATQuant W4A4 linear hot path on B200.

One step = one pass of the whole path over one batch of the Qwen3-8B-shaped
q_proj prefill workload (S=2048 tokens, N=4096, M=4096, bf16 activations):
batq_quant_act (GPK transform + clip + MXFP4 into the tcgen05 scale layout)
followed by batq_gemm_mxfp4 (block-scaled tensor-core GEMM, fp32 out).  The
weights are prepared offline (untimed), as in the method.

Prints one JSON line.  ``value`` is the step's GEMM-equivalent throughput
(2*S*N*M flops per step / device step time, summed over ranks); the per-kernel
numbers (quantiser GB/s, GEMM TFLOP/s, their roofline fractions) ride along.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl batq|reference]

Multi-GPU (torchrun): every rank runs its own batch (weak scaling, no data-path
collective); times are the max over ranks.  ``--impl reference`` times the CPU
oracle on a bounded sample of the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
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
WORKLOAD = "q_proj prefill S=2048 N=4096 M=4096 (Qwen3-8B-shaped), bf16 X, W4A4 MXFP4"
QUANT_BYTES_PER_ELEM = 2 + 0.5 + 1.0 / 32  # bf16 in, E2M1 codes + E8M0 scales out
FP4_NOMINAL_OVER_BF16 = 9.0 / 2.25         # dense fp4 / dense bf16 nominal ratio
ROT = 10                                   # rotating input/output sets (see run_batq)

# DRAM bytes (read + write) per launch from the ncu captures summarised under profiles/, for the
# kernel versions those captures measured; None once a kernel changes until it is re-captured.
NCU_TRAFFIC_BYTES = {
    "k_gemm_pair": 13_585_920,  # read 13,412,864 + write 173,056 B (profiles/k_gemm_pair_q_proj_2048x4096x4096.md)
    "k_quant_act": None,        # counters predate the current quantiser build
}


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
            if self._stop.wait(0.005):
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


def _oracle_step(w, rows, wp):
    from oracle import batq_oracle as O
    x = w.x[rows]
    act = O.quant_act(x, w.A, w.B, w.alpha_min, w.alpha_max)
    out, _ = O.gemm(act["codes"], act["scales"], wp["codes"], wp["scales"])
    return out


def _cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def cpu_baseline(w, wp, budget_s=10.0):
    """Oracle timed on this host: whole steps of the workload (all S tokens) repeated for about
    budget_s seconds, or a row sample of one step when a step alone takes longer."""
    flops_per_row = 2.0 * w.N * w.M
    _oracle_step(w, np.arange(min(64, w.S)), wp)  # first-call overheads stay out of the timing
    t0 = time.perf_counter()
    _oracle_step(w, np.arange(w.S), wp)
    t_step = time.perf_counter() - t0
    if t_step > budget_s:
        rows = int(max(64, w.S * budget_s / t_step))
        t0 = time.perf_counter()
        _oracle_step(w, np.arange(rows), wp)
        dt = time.perf_counter() - t0
        sample = f"{rows} of {w.S} tokens of the q_proj workload"
    else:
        passes, t0 = 0, time.perf_counter()
        while True:
            _oracle_step(w, np.arange(w.S), wp)
            passes += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        dt = time.perf_counter() - t0
        rows = passes * w.S
        sample = f"{passes} whole steps ({w.S} tokens each) of the q_proj workload"
    return {"value": rows * flops_per_row / dt / 1e12, "unit": "TFLOP/s", "cores": _cpu_cores(), "kind": "oracle",
            "sample": f"{sample} (quant_act + fp64 GEMM against all {w.M} prepared weight rows), {dt:.2f} s"}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    from mxfp4_w4a4_post_block_b200 import workloads as WL
    from oracle import batq_oracle as O
    w = WL.q_proj()
    wp = O.prepare_weights(w.W, w.A, w.B)
    t0 = time.perf_counter()
    _oracle_step(w, np.arange(16), wp)
    t_row = (time.perf_counter() - t0) / 16
    rows = int(max(1, min(w.S, 150.0 / (args.steps + args.warmup) / max(t_row, 1e-6))))
    for i in range(args.warmup):
        _oracle_step(w, np.arange(rows), wp)
    times = []
    for i in range(args.steps):
        r0 = (i * rows) % max(1, w.S - rows + 1)
        t0 = time.perf_counter()
        _oracle_step(w, np.arange(r0, r0 + rows), wp)
        times.append(time.perf_counter() - t0)
    t = sum(times) / len(times)
    value = rows * 2.0 * w.N * w.M / t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample_rows_per_step": rows},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _cpu_cores(), "kind": "oracle",
                             "sample": f"{rows} of {w.S} tokens per step"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def per_config(dev, peaks):
    """Kernel-alone throughput on the other workloads (down_proj prefill, decode S=16, the W4A8 and
    NVFP4 variants on q_proj, the seven linears of one S=8192 layer), each timed over back-to-back launches whose inputs rotate through
    more than the 126 MB L2.  Activation codes come from the quantiser; weight codes are random
    bytes with unit scales (timing does not depend on their values)."""
    import torch

    from mxfp4_w4a4_post_block_b200 import batq as BQ
    from mxfp4_w4a4_post_block_b200 import workloads as WL

    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    fp4_peak = peaks["bf16_tflops"] * FP4_NOMINAL_OVER_BF16

    def timed(fns, reps):
        for f in fns:
            f()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            for f in fns:
                f()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / (reps * len(fns))

    def linear_sets(w, copies):
        S, N, M = w.S, w.N, w.M
        X = torch.from_numpy(np.ascontiguousarray(w.x_bits).view(np.int16)).view(torch.bfloat16).to(dev)
        B = torch.from_numpy(np.ascontiguousarray(w.B.reshape(-1))).to(dev)
        ratios = torch.from_numpy(BQ.batq_clip_ratios(w.alpha_min, w.alpha_max)).to(dev)
        g = torch.Generator(device=dev).manual_seed(w.seed)
        out = []
        for c in range(copies):
            codes, scales = BQ.empty_act_buffers(S, N, device=dev)
            wc, wsc = BQ.empty_act_buffers(M, N, device=dev)
            wc.random_(0, 256, generator=g)
            wsc.fill_(127)
            out.append({"X": X if c == 0 else X.clone(), "B": B, "ratios": ratios, "A": w.A, "codes": codes,
                        "scales": scales, "wc": wc, "wsc": wsc, "S": S, "N": N, "M": M,
                        "out": torch.empty((S, M), dtype=torch.float32, device=dev)})
        return out

    def q_fn(z):
        return lambda: BQ.batq_quant_act(z["X"], z["A"], z["B"], z["ratios"], z["codes"], z["scales"],
                                         BQ.BATQ_SCALES_MMA, stream=sp)

    def g_fn(z):
        return lambda: BQ.batq_gemm_mxfp4(z["codes"], z["scales"], z["wc"], z["wsc"], z["S"], z["M"], z["N"],
                                          z["out"], stream=sp)

    res = {}
    # down_proj prefill: S=4096, N=12288, M=4096 (three copies: 300 MB of activations)
    zs = linear_sets(WL.down_proj(with_w=False), 3)
    q_ms = timed([q_fn(z) for z in zs], 10)
    g_ms = timed([g_fn(z) for z in zs], 10)
    S, N, M = zs[0]["S"], zs[0]["N"], zs[0]["M"]
    qb = S * N * QUANT_BYTES_PER_ELEM
    res["down_proj_4096x12288x4096"] = {
        "quant_us": q_ms * 1e3, "quant_gbs": qb / q_ms / 1e6, "quant_frac_hbm": qb / q_ms / 1e6 / peaks["hbm_gbs"],
        "gemm_us": g_ms * 1e3, "gemm_tflops": 2.0 * S * N * M / g_ms / 1e9,
        "gemm_frac_fp4": 2.0 * S * N * M / g_ms / 1e9 / fp4_peak}
    del zs
    # decode: S=16, N=4096, M=24576; the GEMM streams the prepared weights (three copies: 160 MB)
    zs = linear_sets(WL.decode(16, with_w=False), 3)
    q_ms = timed([q_fn(z) for z in zs], 30)
    g_ms = timed([g_fn(z) for z in zs], 30)
    S, N, M = zs[0]["S"], zs[0]["N"], zs[0]["M"]
    lws = [torch.empty(BQ.batq_linear_workspace_size(S, N), dtype=torch.uint8, device=dev) for _ in zs]

    def l_fn(z, ws_buf):
        return lambda: BQ.batq_linear(z["X"], z["A"], z["B"], z["ratios"], z["wc"], z["wsc"], M, ws_buf, z["out"],
                                      stream=sp)

    l_ms = timed([l_fn(z, b) for z, b in zip(zs, lws)], 30)
    wb = M * N * (0.5 + 1.0 / 32)
    res["decode_16x4096x24576"] = {
        "quant_us": q_ms * 1e3, "gemm_us": g_ms * 1e3, "gemm_weight_gbs": wb / g_ms / 1e6,
        "gemm_frac_hbm": wb / g_ms / 1e6 / peaks["hbm_gbs"], "linear_us": l_ms * 1e3,
        "linear_weight_gbs": wb / l_ms / 1e6,
        "note": "launch-bound quantiser (128 KB); GEMM judged on weight bytes against HBM; linear = "
                "batq_linear (the GEMM prefetches its weights into L2 while the quantiser runs)"}
    del zs
    # W4A8 variant on q_proj: MXFP8 activations (3.03 B per element moved) and the E4M3 x E4M3
    # block-scaled GEMM, whose roofline is the dense FP8 rate (measured bf16 x 2)
    w8 = WL.q_proj(with_w=False)
    S, N, M = w8.S, w8.N, w8.M
    X8 = torch.from_numpy(np.ascontiguousarray(w8.x_bits).view(np.int16)).view(torch.bfloat16).to(dev)
    B8 = torch.from_numpy(np.ascontiguousarray(w8.B.reshape(-1))).to(dev)
    r8 = torch.from_numpy(BQ.batq_clip_ratios(w8.alpha_min, w8.alpha_max)).to(dev)
    g8 = torch.Generator(device=dev).manual_seed(7)
    sets8 = []
    for c in range(6):  # 6 x (16.8 MB X + 8.4 + 16.8 MB codes + 33.5 MB out) rotate through L2
        codes8, sc8 = BQ.empty_mxfp8_buffers(S, N, device=dev)
        wc8 = torch.empty((M, N), dtype=torch.uint8, device=dev).random_(0, 128, generator=g8)
        wc8[(wc8 & 0x7F) == 0x7F] = 0x38  # no NaN codes
        _, wsb = BQ.batq_mxfp8_buffer_sizes(M, N)
        sets8.append({"X": X8 if c == 0 else X8.clone(), "codes": codes8, "scales": sc8, "wc": wc8,
                      "wsc": torch.full((wsb,), 127, dtype=torch.uint8, device=dev),
                      "out": torch.empty((S, M), dtype=torch.float32, device=dev)})
    q8 = [lambda z=z: BQ.batq_quant_act_mxfp8(z["X"], w8.A, B8, r8, z["codes"], z["scales"], stream=sp)
          for z in sets8]
    g8f = [lambda z=z: BQ.batq_gemm_w4a8(z["codes"], z["scales"], z["wc"], z["wsc"], S, M, N, z["out"], stream=sp)
           for z in sets8]
    q_ms = timed(q8, 10)
    g_ms = timed(g8f, 10)
    qb = S * N * (2 + 1 + 1.0 / 32)
    fp8_peak = peaks["bf16_tflops"] * 2.0
    res["w4a8_q_proj_2048x4096x4096"] = {
        "quant_us": q_ms * 1e3, "quant_gbs": qb / q_ms / 1e6, "quant_frac_hbm": qb / q_ms / 1e6 / peaks["hbm_gbs"],
        "gemm_us": g_ms * 1e3, "gemm_tflops": 2.0 * S * N * M / g_ms / 1e9,
        "gemm_frac_fp8": 2.0 * S * N * M / g_ms / 1e9 / fp8_peak,
        "note": "MXFP8 activations x MXFP4 weights in E4M3 containers (kind::mxf8f6f4); FP8 peak = measured bf16 x 2"}
    del sets8
    # NVFP4 output on q_proj: E4M3 scale per 16 elements (2.5625 B per element moved; per-tensor
    # encode scale 2.0 from the device) and the kind::mxf4nvf4 GEMM, judged against the FP4 peak
    gsn = torch.full((1,), 2.0, dtype=torch.float32, device=dev)
    gn = torch.Generator(device=dev).manual_seed(11)
    setsn = []
    for c in range(6):  # 6 x (16.8 MB X + 4.2 + 8.4 MB codes + 33.5 MB out) rotate through L2
        cn, sn = BQ.empty_nvfp4_buffers(S, N, device=dev)
        wcn, wsn = BQ.empty_nvfp4_buffers(M, N, device=dev)
        wcn.random_(0, 256, generator=gn)
        wsn.fill_(0x38)  # E4M3 1.0
        setsn.append({"X": X8 if c == 0 else X8.clone(), "codes": cn, "scales": sn, "wc": wcn, "wsc": wsn,
                      "out": torch.empty((S, M), dtype=torch.float32, device=dev)})
    qn = [lambda z=z: BQ.batq_quant_act_nvfp4(z["X"], w8.A, B8, r8, z["codes"], z["scales"], gs=gsn, stream=sp)
          for z in setsn]
    gnf = [lambda z=z: BQ.batq_gemm_nvfp4(z["codes"], z["scales"], gsn, z["wc"], z["wsc"], None, S, M, N, z["out"],
                                          stream=sp) for z in setsn]
    q_ms = timed(qn, 10)
    g_ms = timed(gnf, 10)
    qb = S * N * (2 + 0.5 + 1.0 / 16)
    res["nvfp4_q_proj_2048x4096x4096"] = {
        "quant_us": q_ms * 1e3, "quant_gbs": qb / q_ms / 1e6, "quant_frac_hbm": qb / q_ms / 1e6 / peaks["hbm_gbs"],
        "gemm_us": g_ms * 1e3, "gemm_tflops": 2.0 * S * N * M / g_ms / 1e9,
        "gemm_frac_fp4": 2.0 * S * N * M / g_ms / 1e9 / fp4_peak,
        "note": "NVFP4 activations and weights (E4M3 scale per 16, per-tensor encode scale; kind::mxf4nvf4 block16)"}
    del setsn
    # the seven linears of one S=8192 layer, one after another (each launch reads new inputs)
    zs = []
    for j in range(7):
        zs += linear_sets(WL.layer_linear(j, with_w=False), 1)
    q_ms = timed([q_fn(z) for z in zs], 3) * 7
    g_ms = timed([g_fn(z) for z in zs], 3) * 7
    qb = sum(z["S"] * z["N"] for z in zs) * QUANT_BYTES_PER_ELEM
    fl = sum(2.0 * z["S"] * z["N"] * z["M"] for z in zs)
    res["layer_S8192_7_linears"] = {
        "quant_us": q_ms * 1e3, "quant_gbs": qb / q_ms / 1e6, "quant_frac_hbm": qb / q_ms / 1e6 / peaks["hbm_gbs"],
        "gemm_us": g_ms * 1e3, "gemm_tflops": fl / g_ms / 1e9, "gemm_frac_fp4": fl / g_ms / 1e9 / fp4_peak}
    del zs
    torch.cuda.empty_cache()
    return res


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

    w = WL.q_proj(seed=2 + rank)
    S, N, M = w.S, w.N, w.M
    dev = torch.device("cuda", local)
    X0 = torch.from_numpy(np.ascontiguousarray(w.x_bits).view(np.int16)).view(torch.bfloat16).to(dev)
    B = torch.from_numpy(np.ascontiguousarray(w.B.reshape(-1))).to(dev)
    ratios = torch.from_numpy(BQ.batq_clip_ratios(w.alpha_min, w.alpha_max)).to(dev)
    Wd = torch.from_numpy(w.W).to(dev)
    wc0, wsc0 = BQ.empty_act_buffers(M, N, device=dev)
    pws = torch.empty(BQ.batq_prepare_workspace_size(N), dtype=torch.uint8, device=dev)
    BQ.batq_prepare_weights(Wd, w.A, w.B, wc0, wsc0, pws)
    del Wd, pws
    lws_bytes = BQ.batq_linear_workspace_size(S, N)
    code_bytes = -(-S * (N // 2) // 256) * 256

    # ROT independent sets (activations, prepared weights, workspace, output), visited
    # round-robin: between two uses of a set every other set streams through L2, so each
    # step reads its inputs from HBM (far more than the 126 MB L2 in between).
    sets = []
    for _ in range(ROT):
        ws_buf = torch.empty(lws_bytes, dtype=torch.uint8, device=dev)
        sets.append({
            "X": X0.clone(), "wc": wc0.clone(), "wsc": wsc0.clone(), "lws": ws_buf,
            "codes": ws_buf[:S * (N // 2)].view(S, N // 2), "scales": ws_buf[code_bytes:],
            "out": torch.empty((S, M), dtype=torch.float32, device=dev),
        })
    set_bytes = sum(t.numel() * t.element_size() for t in
                    (sets[0]["X"], sets[0]["wc"], sets[0]["wsc"], sets[0]["lws"], sets[0]["out"]))
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    def step(i):
        # one pass of the whole path: online quantisation + block-scaled GEMM
        # (batq_linear launches the GEMM as a programmatic dependent of the quantiser)
        z = sets[i % ROT]
        BQ.batq_linear(z["X"], w.A, B, ratios, z["wc"], z["wsc"], M, z["lws"], z["out"], stream=sp)

    def quant(i):
        z = sets[i % ROT]
        BQ.batq_quant_act(z["X"], w.A, B, ratios, z["codes"], z["scales"], BQ.BATQ_SCALES_MMA, stream=sp)

    def gemm(i):
        z = sets[i % ROT]
        BQ.batq_gemm_mxfp4(z["codes"], z["scales"], z["wc"], z["wsc"], S, M, N, z["out"], stream=sp)

    def timed(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    warm = max(3, args.warmup)
    for i in range(ROT):
        quant(i)  # every set's workspace holds valid codes before the GEMM-only loop
    for fn in (step, quant, gemm):
        for i in range(warm):
            fn(i)
    torch.cuda.synchronize()
    assert BQ.batq_device_error() == 0

    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        # timed region 1: whole steps back to back (-> value)
        local_ms = timed(step, args.steps)
        # timed region 2: each kernel alone, back to back over the same rotation
        # (-> per-kernel throughput and roofline)
        q_ms = timed(quant, args.steps)
        g_ms = timed(gemm, args.steps)
    if ws > 1:
        dist.barrier()
    local_ms, q_ms, g_ms = max_over_ranks([local_ms, q_ms, g_ms], device=dev)
    assert BQ.batq_device_error() == 0

    # End to end through the public call with host buffers: pinned host X in, fp32 result
    # out, every step.  Copies in both directions run on their own streams so that step
    # i's upload, step i-1's compute and step i-2's download overlap (double-buffered).
    Xh = X0.cpu().pin_memory()
    outh = [torch.empty((S, M), dtype=torch.float32).pin_memory() for _ in range(2)]
    z0 = sets[0]
    Xd = [torch.empty_like(X0) for _ in range(2)]
    outd = [torch.empty((S, M), dtype=torch.float32, device=dev) for _ in range(2)]
    s_up, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    e2e_steps = max(4, min(args.steps, 50))

    def e2e_run(n):
        up = [torch.cuda.Event() for _ in range(n)]
        done = [torch.cuda.Event() for _ in range(n)]
        dn = [torch.cuda.Event() for _ in range(n)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_up)
        stream.wait_event(e0)
        s_dn.wait_event(e0)
        for i in range(n):
            j = i % 2
            if i >= 2:
                s_up.wait_event(done[i - 2])      # Xd[j] no longer read
            with torch.cuda.stream(s_up):
                Xd[j].copy_(Xh, non_blocking=True)
            up[i].record(s_up)
            stream.wait_event(up[i])
            if i >= 2:
                stream.wait_event(dn[i - 2])      # outd[j] already downloaded
            BQ.batq_linear(Xd[j], w.A, B, ratios, z0["wc"], z0["wsc"], M, z0["lws"], outd[j], stream=sp)
            done[i].record(stream)
            s_dn.wait_event(done[i])
            with torch.cuda.stream(s_dn):
                outh[j].copy_(outd[j], non_blocking=True)
            dn[i].record(s_dn)
        s_up.wait_event(dn[n - 1])
        e1.record(s_up)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    e2e_run(3)
    e2e_ms = e2e_run(e2e_steps)
    (e2e_ms,) = max_over_ranks([e2e_ms], device=dev)

    flops = 2.0 * S * N * M
    qbytes = S * N * QUANT_BYTES_PER_ELEM
    peaks = _peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_NOMINAL_OVER_BF16
    gemm_tflops = flops / (g_ms * 1e-3) / 1e12
    quant_gbs = qbytes / (q_ms * 1e-3) / 1e9
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
        "config": {"workload": WORKLOAD, "S": S, "N": N, "M": M,
                   "l2": f"inputs larger than L2: {ROT} rotating sets of X, prepared weights, workspace and "
                         f"output ({ROT * set_bytes / 2**20:.0f} MiB) visited round-robin, steps back to back",
                   "parallelism": f"replicas x{ws} (independent batches)"},
        "quant_gbs": quant_gbs,
        "quant_ms": q_ms,
        "gemm_tflops": gemm_tflops,
        "gemm_ms": g_ms,
        "tokens_per_s": ws * S / (local_ms * 1e-3),
        "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": gemm_tflops / fp4_peak, "traffic": NCU_TRAFFIC_BYTES["k_gemm_pair"],
                     "kernel": "k_gemm_pair",
                     "peak_note": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} x 4 (nominal fp4/bf16)"},
        "roofline_quant": {"bound": "hbm", "achieved": quant_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": quant_gbs / peaks["hbm_gbs"], "traffic": NCU_TRAFFIC_BYTES["k_quant_act"],
                           "kernel": "k_quant_act"},
        "e2e": {"value": whole_job_tflops(ws, flops, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(Xh.numel() * Xh.element_size()),
                "d2h_bytes_per_step": int(outh[0].numel() * outh[0].element_size()), "ms_per_step": e2e_ms,
                "note": "batq_linear on pinned host buffers; upload, compute and download on three streams, "
                        "double-buffered"},
        "gpu_launches": 4 * args.steps,
        "timing": "CUDA events on the launching stream around K back-to-back launches; value: whole steps "
                  "(batq_linear: quantiser + GEMM); per-kernel figures and roofline: K quantiser launches, then K "
                  "GEMM launches, each over the same rotation; gpu_launches counts these three loops",
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_configs:
        line["per_config"] = per_config(dev, peaks)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        from oracle import batq_oracle as O
        wp = O.prepare_weights(w.W, w.A, w.B)
        line["cpu_baseline"] = cpu_baseline(w, wp)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description="BATQuant W4A4 linear benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["batq", "reference"], default="batq")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload kernel timings")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_batq(args)


if __name__ == "__main__":
    sys.exit(main())
