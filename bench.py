"""Benchmark of the online W4A4 rotated linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--tokens M] [--no-cpu-baseline]

One step is one pass of the layer's online hot path over one batch: rotate +
quantize the activations (one kernel) and the W4A4 GEMM with its fused
dequant/outlier epilogue (one kernel).  The weights are rotated and packed
once, offline, before timing (their time is reported separately).  Default
workload: the largest one-GPU layer, the LLaMA-3-70B-shaped FlatQuant gate+up
prefill, X[4096 x 8192] through the Kronecker transform P1 (128x128) kron P2
(64x64) with per-channel scales and clip ratio 0.9, into W[57344 x 8192].

Timing: W warm-up steps, then exactly K steps bracketed by a barrier and a
device synchronize on both sides, CUDA events on the launching stream, max
over ranks.  The timed steps replay CUDA graphs of the two kernels, so the
host's launch cost does not pace the device (it would, for decode-sized
steps of a few microseconds); events between graph replays time each
kernel.  Inputs rotate over several copies whose total exceeds the 126 MB
L2, so no step reads inputs left in L2 by the previous one.  The end-to-end
figure runs the graphed layer through the public API with pinned host
buffers.  Under torchrun each rank runs an independent replica (tokens are
independent; no collective on the data path): weak scaling.

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "W4A4 linear TOPS & rotate+quant GB/s at 1 B200, % of INT8/HBM roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 4.5 / 2.25          # nominal dense INT8 : dense BF16 on B200
DATASHEET_INT8_TOPS = 4500.0


KERNEL_SOURCES = {
    "w4a4_gemm_pair_kernel": ["w4a4_gemm_pair.cu", "qr_device.cuh"],
    "w4a4_gemm_decode_kernel": ["w4a4_gemm_decode.cu", "qr_device.cuh"],
    "w4a4_gemm_decode_kernel_fused": ["w4a4_gemm_decode.cu", "qr_device.cuh", "row_quant.cuh"],
    "wht_ab_kernel": ["rotate_quant.cu", "qr_device.cuh", "row_quant.cuh"],
    "wht_blk_kernel": ["rotate_quant.cu", "qr_device.cuh", "row_quant.cuh"],
    "wht_h12_kernel": ["rotate_quant.cu", "qr_device.cuh", "row_quant.cuh"],
    "wht_few_rows_kernel": ["rotate_quant.cu", "qr_device.cuh", "row_quant.cuh"],
    "kron_tc_kernel": ["kron_tc.cu", "qr_device.cuh"],
    "w8a8_gemm_kernel": ["w8a8_gemm.cu", "qr_device.cuh"],
}
DECODE_MAX_TOKENS = 64          # the GEMM runs its decode kernel up to here


def kernel_source_hash(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        with open(os.path.join(ROOT, "w4a4_rotation_quantized_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def dram_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from the committed ncu capture, or None when the
    capture is missing or the kernel's source has changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(f"{kernel}:{workload}")
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha") != kernel_source_hash(kernel):
        return None
    return rec.get("bytes")


def gemm_kernel_name(M: int, bits: int = 4) -> str:
    if bits == 8:
        return "w8a8_gemm_kernel"
    return "w4a4_gemm_decode_kernel" if M <= DECODE_MAX_TOKENS else "w4a4_gemm_pair_kernel"


def rotate_kernel_name(spec, M: int, sms: int) -> str:
    """The rotate kernel the library routes these (aligned) rows to."""
    if spec.rotation == "kron":
        return "kron_tc_kernel"
    block = spec.block or spec.K
    if M <= sms and not spec.fp4:
        return "wht_few_rows_kernel"
    if block in (64, 128, 256):
        return "wht_blk_kernel"
    if block == 4096 and spec.bits == 4:
        return "wht_h12_kernel"
    return "wht_ab_kernel"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = [("gpu_idle", "nvmlClocksEventReasonGpuIdle"),
               ("applications_clocks", "nvmlClocksEventReasonApplicationsClocksSetting"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("sync_boost", "nvmlClocksEventReasonSyncBoost"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown")]

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []          # (t, sm_mhz, reasons bitmask)
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = nv.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001 - clocks are reported as unavailable
            self.err = repr(e)
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.thread.start()

    def stop(self):
        self._stop.set()
        if self.ok:
            self.thread.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "error": getattr(self, "err", "nvml unavailable")}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed"
        if len(win) < 3:       # very short timed region: widen to the samples around it
            win = [s for s in self.samples if t0 - 0.5 <= s[0] <= t1 + 0.05]
            window = "timed+0.5s before"
        mhz = [s[1] for s in win]
        mask = 0
        for s in win:
            mask |= s[2]
        reasons = [name for name, attr in self.REASONS
                   if getattr(self.nv, attr, 0) and (mask & getattr(self.nv, attr))
                   and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(win), "window": window}


# --------------------------------------------------------------------------- workload

def workload_signs(wl, random_signs: bool, packed_width: int):
    """The seeded random-sign diagonal of a randomized Hadamard over the
    `packed_width` rotated columns (or None).  Each arm sizes it with its own
    implementation's packed width."""
    import workloads
    s = wl.spec
    if not random_signs or s.rotation not in ("hadamard", "gsr"):
        return None
    return workloads.random_signs(s.seed, packed_width)


def oracle_signs(wl, random_signs: bool):
    """workload_signs for the oracle legs (CPU baseline, reference arm)."""
    import oracle as O
    return workload_signs(wl, random_signs,
                          O.packed_width(oracle_rotation(wl), wl.spec.K, wl.spec.n_keep_fp16))


def rotation_for(wl, Q, signs=None):
    s = wl.spec
    import torch
    if s.rotation == "kron":
        return Q.Rotation(Q.KRON, p1=torch.from_numpy(wl.P1).cuda(),
                          p2=torch.from_numpy(wl.P2).cuda(),
                          chan_scale=torch.from_numpy(wl.chan_scale).cuda(),
                          clip_ratio=s.clip_ratio)
    kind = {"hadamard": Q.HADAMARD, "gsr": Q.GSR, "none": Q.NONE}[s.rotation]
    return Q.Rotation(kind, block=s.block, clip_ratio=s.clip_ratio,
                      signs=None if signs is None else torch.from_numpy(signs).cuda())


def oracle_rotation(wl, signs=None):
    import oracle as O
    s = wl.spec
    if s.rotation == "kron":
        return O.Rotation(O.KRON, P1=wl.P1, P2=wl.P2, chan_scale=wl.chan_scale,
                          clip_ratio=s.clip_ratio)
    return O.Rotation({"hadamard": O.HADAMARD, "gsr": O.GSR, "none": O.NONE}[s.rotation],
                      block=s.block, clip_ratio=s.clip_ratio, signs=signs)


def algorithmic_counts(wl, M, kp, asym=False, N=None):
    """Algorithmic work of one step (padding excluded).  Asymmetric activations
    add a zero point per token (written, then read) and a code sum per weight
    row (read).  N overrides the output width (a sample of the weight rows).
    Codes take half a byte each, or one byte in an 8-bit layer."""
    s = wl.spec
    K, N = s.K, (s.N if N is None else N)
    cb = s.bits / 8.0                       # bytes per code
    n_out = s.n_keep_fp16
    k_int = K - n_out
    gemm_ops = 2.0 * M * N * k_int + 2.0 * M * N * n_out
    # rotate+quant: read X, write packed codes, scales (and the fp16 outlier copy)
    rq_bytes = M * K * 2 + M * k_int * cb + M * 4 + M * n_out * 2
    # GEMM: read codes, scales and outlier columns, write Y
    gemm_bytes = (M + N) * k_int * cb + (M + N) * 4 + (M + N) * n_out * 2 + M * N * 2
    if asym:
        rq_bytes += M * 4
        gemm_bytes += (M + N) * 4
    return gemm_ops, rq_bytes, gemm_bytes


def fused_step_bytes(wl, M, kp, asym=False):
    """Algorithmic bytes of one fused decode step (rotate + quantize + GEMM
    in one kernel): the rotate's bytes plus the GEMM's, less the codes,
    scales (zero points) and outlier copy that the GEMM phase reads back
    while they sit in L2 -- X read; codes, scales and the outlier copy
    written; the weight side read; Y written."""
    s = wl.spec
    _, rq_bytes, gemm_bytes = algorithmic_counts(wl, M, kp, asym)
    k_int = s.K - s.n_keep_fp16
    reread = M * k_int * 0.5 + M * 4 + M * s.n_keep_fp16 * 2 + (M * 4 if asym else 0)
    return rq_bytes + gemm_bytes - reread


def kron_split_flops(wl, M):
    """Tensor-core FLOPs of the Kronecker transform of M rows: the two small
    products vec(P1^T mat(x) P2), 2 M K (n1 + n2) FLOPs, three times over for
    the fp16 hi/lo split (hi*hi + hi*lo + lo*hi) that keeps fp32 accuracy."""
    s = wl.spec
    return 3.0 * 2.0 * M * s.K * (s.n1 + s.n2)


def run_ours(args, rank, world, local_rank):
    import torch
    import w4a4_rotation_quantized_b200 as Q
    import workloads
    from w4a4_rotation_quantized_b200 import build as B

    torch.cuda.set_device(local_rank)
    if rank == 0:
        B.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    Q._lib.load()

    wl = workloads.make_workload(args.workload, M=args.tokens)
    s = wl.spec
    M = wl.X.shape[0]
    signs = workload_signs(wl, args.random_signs,
                           Q.packed_k(rotation_for(wl, Q), s.K, s.n_keep_fp16))
    rot = rotation_for(wl, Q, signs)
    idx = None
    if s.n_keep_fp16:
        idx = Q.select_outliers(torch.from_numpy(wl.X_calib).cuda(), s.n_keep_fp16)
    kp = Q.packed_k(rot, s.K, s.n_keep_fp16)
    asym = args.asym_activations
    bits = s.bits
    fp4 = s.fp4
    if (bits == 8 or fp4) and asym:
        raise SystemExit("the 8-bit and FP4 layers take symmetric activations")
    gemm_ops, rq_bytes, gemm_bytes = algorithmic_counts(wl, M, kp, asym)
    # --fused: decode batches run as one kernel (rotate + quantize + GEMM)
    fused = M <= DECODE_MAX_TOKENS and bits == 4 and not fp4 and s.rotation != "kron" and \
        args.fused

    # input sets: enough copies that one pass over them exceeds L2 twice
    x0 = torch.from_numpy(wl.X).cuda()
    w0 = torch.from_numpy(wl.W).cuda()
    t_pack0 = torch.cuda.Event(enable_timing=True)
    t_pack1 = torch.cuda.Event(enable_timing=True)
    Q.QuantizedLinear(w0, rot, idx, asym, bits, fp4, fused)      # warm-up (module load, attributes)
    torch.cuda.synchronize()
    t_pack0.record()
    layer0 = Q.QuantizedLinear(w0, rot, idx, asym, bits, fp4, fused)
    t_pack1.record()
    torch.cuda.synchronize()
    pack_ms = t_pack0.elapsed_time(t_pack1)
    set_bytes = x0.numel() * 2 + layer0.w_codes.numel() + (8 if asym else 4) * s.N + \
        (0 if layer0.w_out is None else layer0.w_out.numel() * 2)
    nsets = max(2, math.ceil(2 * L2_BYTES / set_bytes))
    xs = [x0] + [x0.clone() for _ in range(nsets - 1)]
    wsets = [(layer0.w_codes, layer0.w_scales, layer0.w_out, layer0.w_sums)]
    for _ in range(nsets - 1):
        wsets.append((layer0.w_codes.clone(), layer0.w_scales.clone(),
                      None if layer0.w_out is None else layer0.w_out.clone(),
                      None if layer0.w_sums is None else layer0.w_sums.clone()))
    del w0
    y = torch.empty((M, s.N), dtype=torch.float16, device="cuda")
    stream = torch.cuda.current_stream()

    def rq(x):
        if asym:
            codes, scales, zeros, x_out, _ = Q.rotate_quant_asym(x, rot, idx)
            return codes, scales, x_out, zeros
        if bits == 8:
            codes, scales, x_out, _ = Q.rotate_quant8(x, rot, idx)
            return codes, scales, x_out, None
        if fp4:
            codes, scales, x_out, _ = Q.rotate_quant_fp4(x, rot, idx)
            return codes, scales, x_out, None
        codes, scales, x_out, _ = Q.rotate_quant(x, rot, idx)
        return codes, scales, x_out, None

    def linear(a, wset):
        codes, scales, x_out, zeros = a
        wc, wsc, wo, wsum = wset
        if asym:
            Q.w4a4_linear_asym(codes, scales, zeros, wc, wsc, wsum, x_out, wo, out=y)
        elif bits == 8:
            Q.w8a8_linear(codes, scales, wc, wsc, x_out, wo, out=y)
        elif fp4:
            Q.fp4_linear(codes, scales, wc, wsc, x_out, wo, out=y)
        else:
            Q.w4a4_linear(codes, scales, wc, wsc, x_out, wo, out=y)

    sync = torch.zeros(2, dtype=torch.int32, device="cuda")

    def fused_step(x, wset):
        wc, wsc, wo, wsum = wset
        Q.w4a4_linear_fused(x, rot, idx, wc, wsc, wo, wsum, asym, sync, out=y)

    def step(i):
        if fused:
            fused_step(xs[i % nsets], wsets[i % nsets])
        else:
            linear(rq(xs[i % nsets]), wsets[i % nsets])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # The steps run from CUDA graphs, so that host launch cost does not pace
    # the device: one graph rotates + quantizes G input sets (G = one pass
    # over the sets), another runs the G GEMMs on its outputs.  The timed
    # region replays them in turn; events between replays give each kernel's
    # device time.  A last pair of graphs takes the K mod G remaining steps.
    # (fused: the rotate graph is empty and the second graph runs the fused
    # steps, so its events time the one kernel)
    def rot_pass(n):
        return [] if fused else [rq(xs[i]) for i in range(n)]

    def gemm_pass(outs, n):
        for i in range(n):
            if fused:
                fused_step(xs[i], wsets[i])
            else:
                linear(outs[i], wsets[i])

    def capture(fn):
        if fused and fn is not None and getattr(fn, "rot_side", False):
            return None, fn()                         # nothing to rotate apart
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            r = fn()
        return g, r

    G = nsets
    full, rem = divmod(args.steps, G)
    passes = []
    def rot_fn(n):
        f = lambda: rot_pass(n)
        f.rot_side = True
        return f

    if full:
        g_rot, outs = capture(rot_fn(G))
        g_gemm, _ = capture(lambda: gemm_pass(outs, G))
        passes += [(g_rot, g_gemm)] * full
    if rem:
        g_rot_r, outs_r = capture(rot_fn(rem))
        g_gemm_r, _ = capture(lambda: gemm_pass(outs_r, rem))
        passes.append((g_rot_r, g_gemm_r))
    for gr, gg in set(passes):                        # upload + one untimed replay
        if gr is not None:
            gr.replay()
        gg.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.05)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in passes]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    start.record(stream)
    for (gr, gg), ev in zip(passes, evs):
        ev[0].record(stream)
        if gr is not None:
            gr.replay()
        ev[1].record(stream)
        gg.replay()
        ev[2].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    sampler.stop()
    status = Q._lib.qr_device_status()
    if status != 0:
        raise RuntimeError(f"a kernel reported device status {status:#x}")

    elapsed_ms = start.elapsed_time(end)
    rq_total = sum(e[0].elapsed_time(e[1]) for e in evs)
    gemm_total = sum(e[1].elapsed_time(e[2]) for e in evs)
    elapsed_ms = aggregate_max(elapsed_ms, world)

    # end to end through the public API with host buffers: the graphed layer
    # (host -> its input buffer, replay, its output buffer -> host)
    e2e_steps = min(args.steps, 50)
    x_host = torch.from_numpy(wl.X).pin_memory()
    y_host = torch.empty((M, s.N), dtype=torch.float16).pin_memory()
    glin = Q.GraphedLinear(layer0, M)
    for _ in range(3):
        y_host.copy_(glin(x_host), non_blocking=True)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        y_host.copy_(glin(x_host), non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = aggregate_max(e0.elapsed_time(e1), world) / e2e_steps

    peaks, peak_src = load_peaks()
    if fused:
        gemm_bytes = fused_step_bytes(wl, M, kp, asym)
    ms_per_step = elapsed_ms / args.steps
    value = world * gemm_ops / (ms_per_step * 1e-3) / 1e12
    gemm_avg = gemm_total / args.steps
    rq_avg = rq_total / args.steps
    gemm_tops = gemm_ops / (gemm_avg * 1e-3) / 1e12
    gemm_gbs = gemm_bytes / (gemm_avg * 1e-3) / 1e9
    rq_gbs = rq_bytes / (rq_avg * 1e-3) / 1e9 if rq_avg > 0 else 0.0
    int8_sust = peaks["bf16_tflops_sustained"] * INT8_PER_BF16
    int8_burst = peaks["bf16_tflops"] * INT8_PER_BF16
    timed_s = elapsed_ms * 1e-3
    hbm = peaks["hbm_gbs"]
    clocks = sampler.summary(t0, t1)
    sms = torch.cuda.get_device_properties(local_rank).multi_processor_count
    gemm_name = gemm_kernel_name(M, 8 if fp4 else bits)    # e2m1 runs the pair kernel of the 8-bit codes
    traffic_name = "w4a4_gemm_decode_kernel_fused" if fused else gemm_name
    # the GEMM's bound: tensor cores above the ridge point, HBM below it.
    # The denominator is the burst figure (the timed region is well under a
    # second of GPU time); the sustained and datasheet fractions ride along.
    tensor_bound = gemm_ops / gemm_bytes >= int8_burst * 1e12 / (hbm * 1e9)
    if tensor_bound:
        roofline = {"bound": "tensor", "kernel": gemm_name, "achieved": round(gemm_tops, 1),
                    "peak": round(int8_burst, 1), "unit": "TOP/s",
                    "frac": round(gemm_tops / int8_burst, 4),
                    "peak_source": f"{peak_src} bf16 burst x {INT8_PER_BF16:g} (nominal "
                                   f"INT8:BF16); timed region {timed_s:.3f} s",
                    "frac_of_sustained": round(gemm_tops / int8_sust, 4),
                    "frac_of_datasheet_4500": round(gemm_tops / DATASHEET_INT8_TOPS, 4)}
    else:
        roofline = {"bound": "hbm", "kernel": gemm_name, "achieved": round(gemm_gbs, 1),
                    "peak": hbm, "unit": "GB/s", "frac": round(gemm_gbs / hbm, 4),
                    "peak_source": f"{peak_src} HBM copy bandwidth"}
    roofline.update({"ops_per_launch": gemm_ops, "ms_per_launch": round(gemm_avg, 5),
                     "algorithmic_bytes_per_launch": gemm_bytes,
                     "traffic": dram_traffic(traffic_name, s.name) if M == s.M else None})
    if fused:
        roofline["fused_rotate_quant"] = True
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e2m1" if fp4 else "s8",
        "precision": ("e2m1 codes on the f8f6f4 tensor-core MMA, fp32 accumulate; fp32 rotation; "
                      "fp16 in/out" if fp4 else
                      f"int{bits} codes on s8 tensor-core MMA, s32 accumulate; fp32 rotation; "
                      "fp16 in/out"),
        "data": "synthetic",
        "config": {"workload": s.name, "M": M, "K": s.K, "N": s.N, "K_p": kp,
                   "step": ("one fused kernel (rotate + quantize, grid barrier, GEMM)" if fused
                            else "rotate + quantize kernel, then the GEMM kernel"),
                   "rotation": (("random-sign " if signs is not None else "") +
                                f"{s.rotation}-{s.block}") if s.rotation != "kron"
                   else f"kron-{s.n1}x{s.n2}", "n_out": s.n_keep_fp16,
                   "clip_ratio": s.clip_ratio,
                   "activations": "asymmetric per-token" if asym else "symmetric per-token",
                   "bits": bits,
                   "codes": "e2m1" if fp4 else "int",
                   "parallelism": f"replicas x{world}",
                   "l2": f"inputs rotate over {nsets} copies ({nsets * set_bytes / 1e6:.0f} MB "
                         f"> 126 MB L2)"},
        "roofline": roofline,
        "rotate_quant": ({"fused_into": gemm_name, "bytes_per_launch": rq_bytes,
                          "note": "rotate + quantize run inside the decode kernel, before its "
                                  "grid barrier; their time is part of roofline.ms_per_launch"}
                         if fused else
                         dict(rotate_quant_roofline(wl, M, rq_bytes, rq_avg, peaks, peak_src,
                                                    rotate_kernel_name(s, M, sms)),
                              traffic=dram_traffic(rotate_kernel_name(s, M, sms), s.name)
                              if M == s.M else None)),
        "gemm_hbm_bytes_per_launch": gemm_bytes,
        "offline_weight_pack_ms": round(pack_ms, 3),
        "e2e": {"value": round(world * gemm_ops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TOPS",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": int(x_host.numel() * 2),
                "d2h_bytes_per_step": int(y_host.numel() * 2), "steps": e2e_steps,
                "api": "GraphedLinear"},
        "gpu_launches": (1 if fused else 2) * args.steps,
        "clocks": clocks,
    }
    return result


def rotate_quant_roofline(wl, M, rq_bytes, rq_ms, peaks, peak_src, kernel):
    """Roofline of the rotate+quantize launch.  Hadamard and GSR rows are
    HBM-bound.  The Kronecker transform is bounded by the slower of HBM and
    its split-precision tensor-core FLOPs (fp16 operands, so the bf16 rate);
    frac is the bound's time over the measured time."""
    hbm = peaks["hbm_gbs"]
    sec = rq_ms * 1e-3
    gbs = rq_bytes / sec / 1e9
    out = {"kernel": kernel, "bytes_per_launch": rq_bytes, "ms_per_launch": round(rq_ms, 5),
           "hbm_achieved_gbs": round(gbs, 1), "hbm_peak_gbs": hbm,
           "hbm_frac": round(gbs / hbm, 4)}
    if wl.spec.rotation != "kron":
        out.update({"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(gbs / hbm, 4),
                    "peak_source": f"{peak_src} HBM copy bandwidth"})
        return out
    flops = kron_split_flops(wl, M)
    tfs = flops / sec / 1e12
    t_hbm = rq_bytes / (hbm * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    out.update({"tensor_flops_per_launch": flops, "tensor_achieved_tflops": round(tfs, 1),
                "tensor_peak_tflops": peaks["bf16_tflops"],
                "tensor_frac": round(tfs / peaks["bf16_tflops"], 4)})
    if t_tc >= t_hbm:
        out.update({"bound": "tensor", "achieved": round(tfs, 1), "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": round(t_tc / sec, 4),
                    "peak_source": f"{peak_src} bf16 burst (fp16 operands run at the bf16 rate)"})
    else:
        out.update({"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(t_hbm / sec, 4),
                    "peak_source": f"{peak_src} HBM copy bandwidth"})
    return out


def aggregate_max(value_ms: float, world: int) -> float:
    """Max over ranks of a per-rank duration (device-timed)."""
    if world <= 1:
        return value_ms
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value_ms], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- oracle

def oracle_step(O, asym: bool, bits: int = 4, fp4: bool = False):
    """The oracle's online path: activation quantizer, then the linear."""
    if fp4:
        return lambda x, rot, idx, wside: O.linear_fp4(O.quantize_activations_fp4(x, rot, idx), wside)
    if asym:
        return lambda x, rot, idx, wside: O.linear_asym(
            O.quantize_activations_asym(x, rot, idx), wside)
    return lambda x, rot, idx, wside: O.linear(O.quantize_activations(x, rot, idx, bits), wside)


def _oracle_threads():
    from threadpoolctl import threadpool_info
    return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)


def oracle_sample(workload: str, tokens: int, rows, M_total=None, random_signs: bool = False):
    """The oracle's inputs for a bounded sample of the workload: the first
    `tokens` tokens and the first `rows` weight rows (all of them when rows
    is None), with the weights prepared (offline, untimed)."""
    import oracle as O
    import workloads
    wl = workloads.make_workload(workload, M=M_total, N=rows)
    s = wl.spec
    rot = oracle_rotation(wl, oracle_signs(wl, random_signs))
    idx = O.select_outliers(wl.X_calib, s.n_keep_fp16) if s.n_keep_fp16 else None
    wside = (O.quantize_weights_fp4(wl.W.astype(np.float64), rot, idx) if s.fp4 else
             O.quantize_weights(wl.W.astype(np.float64), rot, idx, s.bits))
    x = wl.X[:tokens].astype(np.float64)
    return wl, rot, idx, wside, x


def oracle_baseline(workload: str, tokens: int, rows, repeats: int = 1, M_total=None,
                    random_signs: bool = False, asym: bool = False, st_tokens: int = 32):
    """Times the CPU oracle's online path on a bounded sample of the workload
    (`tokens` tokens against `rows` weight rows) on the host cores, and once
    more single-threaded on `st_tokens` of those tokens."""
    import oracle as O
    from threadpoolctl import threadpool_limits

    wl, rot, idx, wside, x = oracle_sample(workload, tokens, rows, M_total, random_signs)
    n_rows = wl.W.shape[0]
    run = oracle_step(O, asym, wl.spec.bits, wl.spec.fp4)
    times = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        run(x, rot, idx, wside)
        times.append(time.perf_counter() - t0)
    gemm_ops, _, _ = algorithmic_counts(wl, x.shape[0], 0, N=n_rows)
    sec = statistics.median(times)
    threads = _oracle_threads()
    st = min(st_tokens, x.shape[0])
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        run(x[:st], rot, idx, wside)
        st_sec = time.perf_counter() - t0
    st_ops, _, _ = algorithmic_counts(wl, st, 0, N=n_rows)
    return {"value": round(gemm_ops / sec / 1e12, 6), "unit": "TOPS", "cores": threads,
            "kind": "oracle", "seconds_per_sample": round(sec, 3),
            "sample": f"{x.shape[0]} of {wl.spec.M} tokens x {n_rows} of {wl.spec.N} weight rows "
                      f"of {workload} through the oracle's online path (rotate+quantize+integer "
                      f"GEMM+epilogue), median of {repeats}; weights prepared untimed",
            "single_thread": {"value": round(st_ops / st_sec / 1e12, 6), "unit": "TOPS",
                              "cores": 1, "seconds_per_sample": round(st_sec, 3),
                              "sample": f"{st} tokens x {n_rows} weight rows, one run"}}


def run_reference(args, rank, world):
    """The oracle as the reference arm, on the host cores: each step runs the
    oracle's online path on a bounded sample of the workload."""
    if rank != 0:
        return None
    import oracle as O
    import workloads

    spec = workloads.SPECS[args.workload]
    M_all = args.tokens or spec.M
    tokens = min(M_all, args.reference_tokens)
    rows = min(spec.N, args.reference_rows)
    wl, rot, idx, wside, x = oracle_sample(args.workload, tokens, rows, args.tokens,
                                           args.random_signs)
    s = wl.spec
    run = oracle_step(O, args.asym_activations, s.bits, s.fp4)

    def step():
        run(x, rot, idx, wside)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    sec = (time.perf_counter() - t0) / args.steps
    gemm_ops, _, _ = algorithmic_counts(wl, tokens, 0, N=rows)
    threads = _oracle_threads()
    value = gemm_ops / sec / 1e12
    sample = (f"{tokens} of {M_all} tokens x {rows} of {s.N} weight rows of {s.name} per step "
              f"through the oracle's online path; weights prepared untimed")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": s.name, "M": tokens, "K": s.K, "N": rows,
                   "activations": "asymmetric per-token" if args.asym_activations
                   else "symmetric per-token", "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# --------------------------------------------------------------------------- KV cache

KV_METRIC = "KV-cache R3 + g128 4-bit quantization GB/s at 1 B200, % of HBM"


def kv_bytes(s, tokens):
    """Algorithmic bytes of one KV step: read q, k, v; write q R3, the k and v
    codes (half a byte per value) and a float scale + int32 zero per group."""
    w = s.heads * s.head_dim
    return tokens * w * 2 * 4 + 2 * (tokens * w // 2 + tokens * (w // s.group) * 8)


def run_kv(args, rank, world, local_rank):
    import torch
    import w4a4_rotation_quantized_b200 as Q
    import workloads
    from w4a4_rotation_quantized_b200 import build as B

    torch.cuda.set_device(local_rank)
    if rank == 0:
        B.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    Q._lib.load()
    s, q, k, v = workloads.make_kv(args.workload, args.tokens)
    T = q.shape[0]
    byts = kv_bytes(s, T)
    nsets = max(2, math.ceil(2 * L2_BYTES / (3 * q.nbytes)))
    sets = [tuple(torch.from_numpy(a).cuda() for a in (q, k, v)) for _ in range(nsets)]
    stream = torch.cuda.current_stream()

    def step(i):
        a, b, c = sets[i % nsets]
        return Q.kv_quantize(a, b, c, s.head_dim, s.group)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        keep = [step(i) for i in range(nsets)]
    g.replay()
    torch.cuda.synchronize()
    reps = max(1, args.steps // nsets)
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.05)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    sampler.stop()
    del keep
    if Q._lib.qr_device_status() != 0:
        raise RuntimeError("a kernel reported a device status")
    steps = reps * nsets
    ms = aggregate_max(e0.elapsed_time(e1), world) / steps
    peaks, peak_src = load_peaks()
    gbs = byts / (ms * 1e-3) / 1e9
    # end to end with host buffers: q, k, v in, every output out
    hq, hk, hv = (torch.from_numpy(a).pin_memory() for a in (q, k, v))
    e2e_steps = min(args.steps, 20)
    d_in = [torch.empty_like(t, device="cuda") for t in (hq, hk, hv)]
    r = step(0)
    outs_h = [torch.empty_like(r[0], device="cpu").pin_memory()] + \
        [torch.empty_like(t, device="cpu").pin_memory() for part in r[1:] for t in part]
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a0.record(stream)
    for _ in range(e2e_steps):
        for d, h in zip(d_in, (hq, hk, hv)):
            d.copy_(h, non_blocking=True)
        r = Q.kv_quantize(d_in[0], d_in[1], d_in[2], s.head_dim, s.group)
        flat = [r[0]] + [t for part in r[1:] for t in part]
        for h, d in zip(outs_h, flat):
            h.copy_(d, non_blocking=True)
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = aggregate_max(a0.elapsed_time(a1), world) / e2e_steps
    return {
        "metric": KV_METRIC, "value": round(world * byts / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "precision": "fp16 in, fp32 rotation, 4-bit asymmetric codes + fp32 scale/int32 zero "
                     "per group, fp16 queries out",
        "data": "synthetic",
        "config": {"workload": s.name, "tokens": T, "heads": s.heads, "head_dim": s.head_dim,
                   "group": s.group, "parallelism": f"replicas x{world}",
                   "l2": f"inputs rotate over {nsets} copies"},
        "roofline": {"bound": "hbm", "kernel": "kv_group_quant_kernel + head_rotate_kernel",
                     "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gbs / peaks["hbm_gbs"], 4),
                     "peak_source": f"{peak_src} HBM copy bandwidth",
                     "algorithmic_bytes_per_launch": byts, "traffic": None},
        "e2e": {"value": round(world * byts / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": int(hq.nbytes + hk.nbytes + hv.nbytes),
                "d2h_bytes_per_step": int(sum(h.nbytes for h in outs_h)), "steps": e2e_steps,
                "api": "kv_quantize"},
        "gpu_launches": 3 * steps,
        "clocks": sampler.summary(t0, t1),
    }


def run_kv_reference(args, rank, world):
    """The oracle's KV step on the host cores (rank 0)."""
    if rank != 0:
        return None
    import oracle as O
    import workloads
    s, q, k, v = workloads.make_kv(args.workload, min(args.reference_tokens,
                                                      args.tokens or workloads.KV_SPECS[
                                                          args.workload].tokens))
    q64, k64, v64 = (a.astype(np.float64) for a in (q, k, v))
    for _ in range(args.warmup):
        O.kv_quantize(q64, k64, v64, s.head_dim, s.group)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.kv_quantize(q64, k64, v64, s.head_dim, s.group)
    sec = (time.perf_counter() - t0) / args.steps
    from threadpoolctl import threadpool_info
    threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    value = kv_bytes(s, q.shape[0]) / sec / 1e9
    sample = f"{q.shape[0]} of {s.tokens} tokens of {s.name} per step through the oracle"
    return {
        "impl": "reference", "metric": KV_METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": s.name, "tokens": q.shape[0], "heads": s.heads,
                   "head_dim": s.head_dim, "group": s.group, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# --------------------------------------------------------------------------- main

def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="flatquant_gate_up_8192")
    ap.add_argument("--tokens", type=int, default=None, help="override the token count M")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-baseline-tokens", type=int, default=512)
    ap.add_argument("--cpu-baseline-rows", type=int, default=8192,
                    help="weight rows in the CPU baseline's sample (capped at N)")
    ap.add_argument("--reference-tokens", type=int, default=64)
    ap.add_argument("--reference-rows", type=int, default=4096,
                    help="weight rows in the reference arm's per-step sample (capped at N)")
    ap.add_argument("--random-signs", action="store_true",
                    help="randomized Hadamard: a seeded random-sign diagonal before the blocks")
    ap.add_argument("--fused", action="store_true",
                    help="decode batches (<= 64 tokens): time the fused decode kernel (rotate + "
                         "quantize + GEMM in one launch) instead of the two launches")
    ap.add_argument("--asym-activations", action="store_true",
                    help="QUIK's asymmetric per-token activation quantizer (zero point per token)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")

    import workloads
    kv = args.workload in workloads.KV_SPECS
    if args.impl == "reference":
        res = run_kv_reference(args, rank, world) if kv else run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_kv(args, rank, world, local_rank) if kv else run_ours(args, rank, world,
                                                                         local_rank)
        if rank == 0 and kv and world == 1 and not args.no_cpu_baseline:
            ref = run_kv_reference(argparse.Namespace(
                workload=args.workload, tokens=args.tokens, reference_tokens=64, warmup=1,
                steps=3), 0, 1)
            res["cpu_baseline"] = ref["cpu_baseline"]
            print(json.dumps(res), flush=True)
        elif rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                tokens = min(args.cpu_baseline_tokens, res["config"]["M"])
                rows = min(args.cpu_baseline_rows, res["config"]["N"])
                res["cpu_baseline"] = oracle_baseline(args.workload, tokens, rows, repeats=3,
                                                      M_total=args.tokens,
                                                      random_signs=args.random_signs,
                                                      asym=args.asym_activations)
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
