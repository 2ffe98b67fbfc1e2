#!/usr/bin/env python
"""Benchmark: OmniQuant fake-quantized linear calibration steps per second on B200.

A step is one pass of the whole hot path over one calibration batch: LET (activation and
weight side), LWC fake-quant of the weight, per-token activation fake-quant (when
configured), the tcgen05 forward GEMM with the fused bias / MSE / dY epilogue, the
straight-through backward (dW^ and dXq GEMMs, STE reductions, LET gradients) and the AdamW
update, all through one omq_calib_step call on one stream. Inputs are synthetic and
resident in HBM when the timed region starts. The default workload is the largest
single-layer case, the LLaMA-13B down_proj shape (2048 tokens x 13824 -> 5120, W2A16, group
64, no LET: the layer's input follows the FFN nonlinearity); the q_proj (W4A16 g128, LET),
gate/up (W4A4 per-channel, LET) and whole-block workloads run with --config.

One process per GPU (torchrun for N > 1): each rank calibrates its own independent layer
(different seed), with no collective on the data path; the timed region is bracketed by a
barrier and device synchronisation and its length is the maximum over ranks.

Also printed on the same JSON line: the roofline of the dominant kernel (the tcgen05 GEMM,
timed with CUDA events around its launches inside the timed region), the CPU oracle timed
on the host as a reported baseline, an end-to-end figure through the same C ABI with the
step's inputs copied from pinned host memory inside the timed region, and the SM clocks
sampled during the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fake-quant linear fwd+bwd calib steps/s; TFLOP/s & GB/s as % of roofline"
UNIT = "steps/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="llama13b_down_w2a16g64")
    ap.add_argument("--impl", default="omq", choices=["omq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in ("gemm_tc.cu", "gemm_epilogue.cuh", "omq_internal.cuh"):
        with open(os.path.join(ROOT, "post_quantization_lwc_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the GEMM kernel from a committed ncu summary, when the kernel
    source has not changed since the counters were taken; otherwise None."""
    path = os.path.join(ROOT, "profiles", "gemm_tc_traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("source_sha") != kernel_source_hash():
        return None
    return rec.get("bytes_per_launch", {}).get(workload)


def bind_host_to_gpu(dev_index: int) -> str:
    """Pin this process to the CPUs NVML reports as local to the GPU (its PCIe root's NUMA
    node) before any pinned host buffer is allocated, so host-to-device copies come from
    local memory. Changes only this process's CPU affinity; no GPU setting. Returns a note."""
    try:
        import pynvml
        import torch
        uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
        pynvml.nvmlInit()
        try:
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            words = pynvml.nvmlDeviceGetCpuAffinity(h, (os.cpu_count() + 63) // 64)
        finally:
            pynvml.nvmlShutdown()
        cpus = {64 * i + b for i, w in enumerate(words) for b in range(64) if (int(w) >> b) & 1}
        cpus &= os.sched_getaffinity(0)
        if not cpus:
            return "unbound (no GPU-local CPU available)"
        os.sched_setaffinity(0, cpus)
        return f"{len(cpus)} GPU-local CPUs (NVML affinity)"
    except Exception as e:  # noqa: BLE001 - the binding is an optimisation, never required
        return f"unbound ({type(e).__name__})"


def run_e2e(step, hosts, loss, steps: int, dev):
    """Whole steps through the public API from pinned host memory: each step's inputs are
    copied host -> device on a copy stream into one of two device buffer sets (step i + 1's
    upload overlaps step i's compute; a buffer set is refilled only after the step that read
    it), the step runs on the compute stream once its copy has landed, and its loss is read
    back into pinned host memory. Returns the elapsed milliseconds, CUDA events on the
    compute stream; every copy lies between the two events."""
    import torch
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream(device=dev)
    bufs = [[torch.empty(h.shape, dtype=h.dtype, device=dev) for h in hosts] for _ in range(2)]
    lh = torch.empty(steps, dtype=torch.float32).pin_memory()
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    start = torch.cuda.Event()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(comp)
    start.record(comp)
    for c in consumed:
        c.record(comp)
    copy.wait_event(start)

    def upload(i):
        b = i % 2
        copy.wait_event(consumed[b])
        with torch.cuda.stream(copy):
            for d, h in zip(bufs[b], hosts):
                d.copy_(h, non_blocking=True)
        copied[b].record(copy)

    upload(0)
    for i in range(steps):
        if i + 1 < steps:
            upload(i + 1)
        b = i % 2
        comp.wait_event(copied[b])
        step(*bufs[b])
        consumed[b].record(comp)
        lh[i:i + 1].copy_(loss.reshape(1), non_blocking=True)
    e1.record(comp)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def step_flops(cfg) -> int:
    """Dense contractions of one step: forward, dW^ and (LET learnable) dXq GEMMs."""
    n_gemm = 3 if cfg.let else 2
    return n_gemm * 2 * cfg.m_tokens * cfg.n_out * cfg.k_in


def phase_bytes(cfg) -> dict:
    """Algorithmic DRAM bytes of the memory-bound phases of omq_calib_step as the step runs them
    (16-bit storage, float16 GEMM operands, the weight-side STE fused into the dW^ GEMM, B~
    fused into the LWC pass): every tensor a phase must read or write, once. The GEMM phases
    are counted in flops instead."""
    es = 4 if cfg.dtype == "f32" else 2          # storage of W and X
    op = 4 if cfg.dtype == "f32" else 2          # GEMM operands Xq, W^, dY
    M, N, K, ng = cfg.m_tokens, cfg.n_out, cfg.k_in, cfg.n_groups
    grp = N * ng
    rec = 4 + 4 + 16                             # h, z, range record
    out = {}
    # activation side of the forward: X~ (LET), per-token act quant, or the operand conversion
    if cfg.let or cfg.abits < 16:   # otherwise X itself is the GEMM operand: no pass
        out["let"] = es * M * K + op * M * K + (M * rec if cfg.abits < 16 else 0)
    # W, logits (and s, delta) in; W^, h, z, ranges (and B~) out
    out["lwc"] = es * N * K + 8 * grp + op * N * K + rec * grp + (8 * K + 4 * N if cfg.let else 0)
    if cfg.let:
        # dB~: column sums of dY, then the 64-row partials reduced
        out["dbias"] = op * M * N + 2 * 4 * -(-M // 64) * N
    if op == 2 and cfg.group % 32 == 0:
        # fused path: finish reads the per-32-column partials and the group records, writes the
        # logit gradients and the extremes' shares; with LET the correction pass reads W again
        fin = 2 * 4 * N * (K // 32) + grp * (4 + 16 + 8) + grp * 8 + (grp * 8 if cfg.let else 0)
        corr = (es * N * K + grp * (16 + 8) + 4 * N + 2 * 4 * -(-N // 32) * K) if cfg.let else 0
        out["ste_w"] = fin + corr
    else:
        out["ste_w"] = 4 * N * K + es * N * K + grp * (rec + 8 + 8)
    if cfg.let:
        # X and the float32 dXq in, per-64-token column partials of d s and d delta out
        out["ste_x"] = es * M * K + 4 * M * K + 2 * 4 * -(-M // 64) * K + \
            (M * rec if cfg.abits < 16 else 0)
    return out


class ClockSampler(threading.Thread):
    """Polls NVML for the SM clock and the clock-event reasons while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.005):
        super().__init__(daemon=True)
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.ok = False
        self.uuid = None
        self._halt = threading.Event()
        try:
            import pynvml
            import torch
            # NVML numbers the node's GPUs without regard to CUDA_VISIBLE_DEVICES: resolve
            # the CUDA device by its UUID so the samples come from the GPU this process uses
            uuid = str(torch.cuda.get_device_properties(index).uuid)
            self.uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def run(self):
        if not self.ok:
            return
        while not self._halt.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._halt.set()
        self.join(timeout=2)

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": getattr(self, "max_mhz", None), "reasons": [],
                    "samples": 0, "gpu_uuid": self.uuid}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b and b != 0x1],
                "samples": len(self.samples), "gpu_uuid": self.uuid}


def workload_config(cfg):
    return {"workload": cfg.name, "M_tokens": cfg.m_tokens, "K_in": cfg.k_in, "N_out": cfg.n_out,
            "group": cfg.group, "bits": cfg.bits, "abits": cfg.abits, "let": cfg.let,
            "storage": cfg.dtype}


# ----------------------------------------------------------------------------- oracle (CPU)

def oracle_sample(cfg, inp, rows: int | None):
    """A bounded sample of the workload for the CPU oracle: the first `rows` output rows
    (the whole layer when None). Returns numpy inputs and the fraction of the layer."""
    import numpy as np

    from oracle import omniquant as om
    from post_quantization_lwc_b200 import synth
    X = synth.as_f32_numpy(inp.X)
    W = synth.as_f32_numpy(inp.W)
    n = cfg.n_out if rows is None else rows
    W = np.ascontiguousarray(W[:n])
    Yref = om.reference_output(X, W, inp.B.numpy()[:n]).astype(np.float32)
    return dict(X=X, W=W, B=inp.B.numpy()[:n], Yref=Yref, gl=inp.gamma_logit.numpy()[:n],
                bl=inp.beta_logit.numpy()[:n], s=inp.s.numpy(), d=inp.delta.numpy()), n / cfg.n_out


def oracle_steps(cfg, smp, steps: int):
    from oracle import omniquant as om
    return om.calibrate(smp["X"], smp["W"], smp["B"], smp["Yref"], smp["gl"], smp["bl"], smp["s"],
                        smp["d"], cfg.bits, cfg.group, cfg.abits, cfg.let, steps)


def blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cfg, inp, budget_s: float = 20.0):
    """Time the oracle (as it stands) on the host: whole steps of the full layer while they
    fit the budget, else a row sample scaled to the layer."""
    smp, frac = oracle_sample(cfg, inp, None)
    t0 = time.perf_counter()
    oracle_steps(cfg, smp, 1)
    t1 = time.perf_counter() - t0
    steps = max(1, min(5, int(budget_s / max(t1, 1e-3)) - 1))
    t0 = time.perf_counter()
    oracle_steps(cfg, smp, steps)
    dt = time.perf_counter() - t0
    return {"value": steps * frac / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{steps} whole calibration step(s) of the full {cfg.name} layer "
                      f"(numpy binary64 oracle, after one untimed step), {dt:.1f} s"}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, cfg, rank: int, world: int):
    if rank != 0:
        return 0
    from post_quantization_lwc_b200 import synth
    inp = synth.make_inputs(cfg)
    smp, frac = oracle_sample(cfg, inp, None)
    t0 = time.perf_counter()
    oracle_steps(cfg, smp, 1)
    t1 = time.perf_counter() - t0
    total = (args.steps + args.warmup) * t1
    rows = None
    if total > 150.0:   # keep the whole run within a few minutes: sample output rows
        rows = max(8, int(cfg.n_out * 150.0 / total) // 8 * 8)
        smp, frac = oracle_sample(cfg, inp, rows)
    if args.warmup > 1:
        oracle_steps(cfg, smp, args.warmup - 1)
    t0 = time.perf_counter()
    oracle_steps(cfg, smp, args.steps)
    dt = time.perf_counter() - t0
    value = args.steps * frac / dt
    sample = (f"whole {cfg.name} layer per step" if rows is None else
              f"first {rows} of {cfg.n_out} output rows per step, throughput scaled by "
              f"{cfg.n_out}/{rows}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {**workload_config(cfg), "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- libomq arm

def run_omq(args, cfg, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    from post_quantization_lwc_b200 import omq, synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    host_note = bind_host_to_gpu(local_rank)
    import dataclasses
    my_cfg = dataclasses.replace(cfg, seed=cfg.seed + 1000 * rank) if rank else cfg
    inp = synth.make_inputs(my_cfg)
    dt = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
    lc = omq.LinearCalibration(M=cfg.m_tokens, N=cfg.n_out, K=cfg.k_in, group=cfg.group,
                               bits=cfg.bits, abits=cfg.abits, let=cfg.let, dtype=dt, device=dev)
    lc.load(inp.W.to(dev), inp.gamma_logit.to(dev), inp.beta_logit.to(dev), s=inp.s.to(dev),
            delta=inp.delta.to(dev), B=inp.B.to(dev))
    X = inp.X.to(dev).contiguous()
    Yref = lc.reference_output(X).contiguous()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        lc.step(X, Yref)
    torch.cuda.synchronize()
    omq.sync_check()

    # per-phase split: an eager pass with CUDA events at the phase boundaries
    n_ph = min(args.steps, 20)
    timer = omq.PhaseTimer(n_ph)
    for i in range(n_ph):
        lc.step(X, Yref, events=timer.sets[i])
    torch.cuda.synchronize()
    phases = timer.mean_ms()

    # the timed region: the K steps captured once as a CUDA graph (one launch sequence, no
    # host work between kernels), replayed once to warm it and once under the clock
    graph, cap_stream = torch.cuda.CUDAGraph(), torch.cuda.Stream()
    cap_stream.wait_stream(torch.cuda.current_stream())
    n0 = omq.launch_count()
    with torch.cuda.stream(cap_stream):
        with torch.cuda.graph(graph, stream=cap_stream):
            for _ in range(args.steps):
                lc.step(X, Yref)
    n1 = omq.launch_count()
    graph.replay()
    torch.cuda.synchronize()
    omq.sync_check()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    ev0.record()
    graph.replay()
    ev1.record()
    torch.cuda.synchronize()
    sampler.stop()
    barrier()
    omq.sync_check()
    ms = ev0.elapsed_time(ev1)
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    last_loss = float(lc.loss.item())

    # end to end through the same C ABI: each step's X and Y* come from pinned host memory
    e2e = None
    if not args.no_e2e:
        # the step's input is the calibration batch X; its target Y* = X W^T + B is the
        # full-precision layer's output, recomputed on the device every step (library GEMM)
        Xh = inp.X.pin_memory()
        barrier()
        ems = run_e2e(lambda x: lc.step(x, lc.reference_output(x)), [Xh], lc.loss, args.steps,
                      dev)
        barrier()
        if world > 1:
            t = torch.tensor([ems], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        e2e = {"value": world * args.steps / (ems / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": Xh.numel() * Xh.element_size(),
               "target": "Y* = X W^T + B, the full-precision layer's output, computed on the "
                         "device from the uploaded X every step (omq_fq_linear_fwd, inside "
                         "the timed region)",
               "d2h_bytes_per_step": 4,
               "overlap": "double-buffered inputs: step i+1's host-to-device copy (copy "
                          "stream) runs under step i (compute stream)",
               "host": host_note}

    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    op_name = {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}[lc.op_dtype]
    value = world * args.steps / (ms / 1e3)
    gemm_keys = ["fwd_gemm", "dw_gemm"] + (["dx_gemm"] if cfg.let else [])
    gemm_ms = sum(phases[k] for k in gemm_keys) / len(gemm_keys)
    gemm_flops = 2 * cfg.m_tokens * cfg.n_out * cfg.k_in
    achieved = gemm_flops / (gemm_ms * 1e-3) / 1e12
    timed_s = ms / 1e3
    peak_key = "bf16_tflops" if timed_s < 1.0 else "bf16_tflops_sustained"
    peak = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    pbytes = phase_bytes(cfg)
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    phase_report = {}
    for k in omq.PHASES:
        entry = {"us": round(phases[k] * 1e3, 2)}
        if k in pbytes and phases[k] > 0.0005 and pbytes[k] > 0:
            gbs = pbytes[k] / (phases[k] * 1e-3) / 1e9
            entry.update({"gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm, 3)})
        if k in gemm_keys:
            tf = gemm_flops / (phases[k] * 1e-3) / 1e12
            entry.update({"tflops": round(tf, 1), "tc_frac": round(tf / peak, 3)})
        phase_report[k] = entry
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": op_name,
        "dtype_detail": (f"{cfg.dtype} storage of W and X; {op_name} GEMM operands (Xq, W^, "
                         "dY) with float32 accumulation; float32 quantizer, STE and AdamW "
                         "arithmetic" if cfg.dtype == "bf16" else "float32 throughout"),
        "data": "synthetic (seeded LLaMA-shaped weights and outlier-channel activations)",
        "config": {**workload_config(cfg),
                   "l2": "no flush: the step's working set (W, W^, X, Xq, Y*, dY, dW^, dXq) "
                         "exceeds the 126 MB L2",
                   "parallelism": f"replicas x{world} (one independent layer per GPU)"},
        "tflops": step_flops(cfg) * value / 1e12,
        "roofline": {"bound": "tensor", "kernel": "gemm_tc_kernel", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": recorded_traffic(cfg.name),
                     "peak_source": f"{peak_key} of {peak_src}",
                     "per_launch": f"2*M*N*K = {gemm_flops / 1e9:.1f} GFLOP over the average "
                                   f"duration of the {len(gemm_keys)} GEMM launches per step"},
        "phases": phase_report,
        "loss": last_loss,
        "gpu_launches": int(n1 - n0),
        "timing": "K steps replayed from one CUDA graph; phases from a separate eager pass "
                  "with CUDA events at the phase boundaries",
        "clocks": sampler.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, inp)
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- block workload

def block_flops(bc) -> dict:
    """Dense contractions of one block step: the seven linears (forward, dW^, dXq each; the
    q/k/v and gate/up linears as one [3D, D] and one [2I, D] weight), and the six attention
    products with only the causal lower triangle counted (half of each M x M product)."""
    M, D, H, I = bc.M, bc.D, bc.H, bc.I
    lin = 3 * 2 * M * (3 * D * D + D * D + 2 * I * D + D * I)
    attn = 6 * 2 * M * M * 128 * H // 2
    return {"linears": lin, "attention": attn, "total": lin + attn}


def block_oracle_sample(bc, tokens: int):
    """The oracle's block step on the first `tokens` tokens of the workload (full weights)."""
    import numpy as np

    from oracle import block as ob
    from post_quantization_lwc_b200 import synth
    inp = synth.make_block_inputs(bc)
    sh = ob.BlockShape(M=tokens, D=bc.D, H=bc.H, I=bc.I, wbits=bc.wbits, abits=bc.abits,
                       group=bc.group)
    x = synth.as_f32_numpy(inp.x[:tokens])
    W = {k: synth.as_f32_numpy(v) for k, v in inp.W.items()}
    theta = synth.init_block_theta(bc, ob.theta_layout(sh)).numpy()
    y_ref = ob.block_reference(sh, x, W)
    return sh, x, W, theta, y_ref


def block_cpu_time(bc, tokens: int, steps: int):
    from oracle import block as ob
    sh, x, W, theta, y_ref = block_oracle_sample(bc, tokens)
    t0 = time.perf_counter()
    for _ in range(steps):
        ob.block_step(sh, x, W, theta, y_ref)
    return time.perf_counter() - t0


def block_cpu_baseline(bc, tokens: int = 128, steps: int = 1):
    """The oracle (as it stands) on a bounded sample: whole block steps on the first `tokens`
    tokens with the full weights, throughput scaled to the workload by the step's flops."""
    dt = block_cpu_time(bc, tokens, steps)
    import dataclasses
    small = dataclasses.replace(bc, M=tokens)
    scale = block_flops(small)["total"] / block_flops(bc)["total"]
    return {"value": steps * scale / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{steps} block step(s) of the numpy binary64 oracle on the first {tokens} "
                      f"of {bc.M} tokens with the full {bc.name} weights ({dt:.1f} s), "
                      f"throughput scaled by the flop ratio {scale:.4f}"}


def run_block_reference(args, bc, rank: int, world: int):
    if rank != 0:
        return 0
    tokens = 128
    t1 = block_cpu_time(bc, tokens, 1)
    if args.warmup > 1:
        block_cpu_time(bc, tokens, min(args.warmup - 1, 2))
    steps = max(1, min(args.steps, int(120.0 / max(t1, 1e-3))))
    dt = block_cpu_time(bc, tokens, steps)
    import dataclasses
    scale = block_flops(dataclasses.replace(bc, M=tokens))["total"] / block_flops(bc)["total"]
    value = steps * scale / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {**block_config(bc), "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": f"{steps} oracle block step(s) on the first {tokens} "
                                       f"tokens, scaled by the flop ratio {scale:.4f}"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def block_config(bc):
    return {"workload": bc.name, "M_tokens": bc.M, "hidden": bc.D, "heads": bc.H,
            "ffn": bc.I, "group": bc.group or "per-channel", "bits": bc.wbits,
            "abits": bc.abits, "let": "all linears but down; Q/K affinity", "storage": "bf16"}


def run_block(args, bc, rank: int, world: int, local_rank: int):
    import dataclasses

    import torch
    import torch.distributed as dist

    from post_quantization_lwc_b200 import omq, synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    host_note = bind_host_to_gpu(local_rank)
    my = dataclasses.replace(bc, seed=bc.seed + 1000 * rank) if rank else bc
    inp = synth.make_block_inputs(my)
    blk = omq.Block(bc.M, bc.D, bc.H, bc.I, group=bc.group, wbits=bc.wbits, abits=bc.abits,
                    device=dev)
    names = [(n, blk.theta_slices[n][1]) for n in omq.THETA]
    blk.load({k: v.to(dev) for k, v in inp.W.items()}, synth.init_block_theta(bc, names).to(dev))
    x = inp.x.to(dev).contiguous()
    y_ref = blk.reference(x).contiguous()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        blk.step(x, y_ref)
    torch.cuda.synchronize()
    omq.sync_check()
    nph = len(omq.BLOCK_PHASES)
    n_ph = min(args.steps, 10)
    sets = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 1)] for _ in range(n_ph)]
    for es in sets:
        for e in es:
            e.record()
    for i in range(n_ph):
        blk.step(x, y_ref, events=sets[i])
    torch.cuda.synchronize()
    phases = {p: sum(es[j].elapsed_time(es[j + 1]) for es in sets) / n_ph
              for j, p in enumerate(omq.BLOCK_PHASES)}
    graph, cap_stream = torch.cuda.CUDAGraph(), torch.cuda.Stream()
    cap_stream.wait_stream(torch.cuda.current_stream())
    n0 = omq.launch_count()
    with torch.cuda.stream(cap_stream):
        with torch.cuda.graph(graph, stream=cap_stream):
            for _ in range(args.steps):
                blk.step(x, y_ref)
    n1 = omq.launch_count()
    graph.replay()
    torch.cuda.synchronize()
    omq.sync_check()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    ev0.record()
    graph.replay()
    ev1.record()
    torch.cuda.synchronize()
    sampler.stop()
    barrier()
    omq.sync_check()
    ms = ev0.elapsed_time(ev1)
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())

    e2e = None
    if not args.no_e2e:
        xh = inp.x.pin_memory()
        yh = y_ref.cpu().pin_memory()
        barrier()
        ems = run_e2e(lambda a, b: blk.step(a, b), [xh, yh], blk.loss, args.steps, dev)
        barrier()
        if world > 1:
            t = torch.tensor([ems], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        e2e = {"value": world * args.steps / (ems / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": xh.numel() * xh.element_size() + yh.numel() * yh.element_size(),
               "d2h_bytes_per_step": 4,
               "overlap": "double-buffered inputs: step i+1's host-to-device copy (copy "
                          "stream) runs under step i (compute stream)",
               "host": host_note}
    if rank != 0:
        return 0
    peaks, peak_src = load_peaks()
    value = world * args.steps / (ms / 1e3)
    fl = block_flops(bc)
    step_s = ms / 1e3 / args.steps
    peak_key = "bf16_tflops" if ms / 1e3 < 1.0 else "bf16_tflops_sustained"
    peak = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    achieved = fl["total"] / step_s / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded LLaMA-7B-shaped block weights, outlier-channel inputs)",
        "config": {**block_config(bc),
                   "l2": "no flush: the step's working set (weights, scores, probabilities) "
                         "exceeds the 126 MB L2",
                   "parallelism": f"replicas x{world} (one independent block per GPU)"},
        "tflops": fl["total"] * value / 1e12,
        "roofline": {"bound": "tensor", "kernel": "whole step (tcgen05 GEMMs dominate)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "peak_source": f"{peak_key} of {peak_src}",
                     "per_launch": f"{fl['total'] / 1e9:.0f} GFLOP per step (linears "
                                   f"{fl['linears'] / 1e9:.0f}, causal attention "
                                   f"{fl['attention'] / 1e9:.0f}) over the step time"},
        "phases_ms": {k: round(v, 4) for k, v in phases.items()},
        "loss": float(blk.loss.item()),
        "gpu_launches": int(n1 - n0),
        "timing": "K steps replayed from one CUDA graph; phases from a separate eager pass "
                  "with CUDA events at the phase boundaries",
        "clocks": sampler.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = block_cpu_baseline(bc)
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    from post_quantization_lwc_b200 import synth
    if args.config in synth.BLOCK_CONFIGS:
        bc = synth.BLOCK_CONFIGS[args.config]
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        if args.impl == "reference":
            return run_block_reference(args, bc, rank, world)
        if world > 1:
            import torch
            import torch.distributed as dist
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local_rank))
        try:
            return run_block(args, bc, rank, world, local_rank)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
    cfg = synth.CONFIGS[args.config]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, cfg, rank, world)
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_omq(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
