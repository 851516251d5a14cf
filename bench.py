#!/usr/bin/env python3
"""Benchmark of the ConvRot W4A4 quantized Linear on B200.

One *step* is one pass of the whole hot path over one batch of synthetic
input: for every linear of the workload, the fused ConvRot W4A4 Linear
(online rotation + per-token INT4 quantization, then the tensor-core W4A4
GEMM with the rank-one scale + bias epilogue, bf16 out).

Default workload (``edit20b``, the largest single-GPU configuration): the
linears of one block of the 20B-class image-edit DiT, 8192 image + 512 text
tokens (M = 8704), hidden 3072: to_q/k/v/out (3072 -> 3072), MLP up (3072 ->
12288) and down (12288 -> 3072).  Other workloads: ``qwen3_4b`` (the Qwen3-4B
text-encoder layer at M = 76 and 1220), ``dit6b`` (M = 4224, hidden 3840),
``small_m`` (M in 1..128), ``small``, and the int8 / asymmetric W4A8 ones.

Metric: effective TOPS = sum over the step's linears of 2*M*N*K / step time.
The line also carries ``small_m``: HBM GB/s of the fused Linear and of the
GEMM at M in {1, 8, 16} (the bandwidth-bound regime), each a steady-state
per-call time over back-to-back calls on distinct weight copies.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
        [--workload NAME] [--no-e2e]
Multi-GPU: every rank (one per GPU) runs the same workload (replicas, weak
scaling, no data-path collective); the time is the max over ranks.  Under
torchrun the ranks come from the environment; ``--gpus N`` without torchrun
starts the N ranks itself.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "ConvRot W4A4 linear effective TOPS & % INT8-TC peak; HBM GB/s at M<=16"
UNIT = "TOPS"
WORKLOAD_DESC = {
    "qwen3_4b": "Qwen3-4B text-encoder layer linears (q,k,v,o,gate,up,down; hidden 2560) at M=76 and M=1220",
    "dit6b": "6B DiT block linears at 1024x1024 (qkv, out, ffn up, ffn down; hidden 3840), M=4224",
    "edit20b": "20B image-edit DiT linears (to_q/k/v/out, mlp up/down; hidden 3072), M=8704",
    "small_m": "small-M sweep, M in {1,8,16,64,128} x (K,N) in {(2560,9728),(9728,2560),(3072,12288),(12288,3072)}",
    "small": "single linear M=32, K=512, N=256",
    "edit20b_int8": "20B image-edit DiT value/output projections (3072x3072) in int8_tensorwise W8A8, M=8704",
    "qwen3_4b_mixed": "Qwen3-4B layer at M=76 and M=1220: q,k,v,o in ConvRot INT8 (row-scaled) W8A8, "
                      "gate,up,down in ConvRot W4A4",
    "qwen3_4b_w4a8": "Qwen3-VL-4B text-encoder layer linears (q,k,v,o,gate,up,down; hidden 2560) in asymmetric "
                     "W4A8 (4-bit codebook weights, e4m3 group-16 scales), M=76 and M=1220",
    "small_m_w4a8": "small-M sweep in asymmetric W4A8, M in {1,8,16,64,128} x (K,N) in {(2560,9728),(9728,2560),"
                    "(3072,12288),(12288,3072)}",
}
# w8a8_format_t of each 8-bit-activation format's quantizer (the asymmetric
# W4A8 activations are the ConvRot INT8 row-scaled codes)
FORMAT_ID = {"int8_tensorwise": 0, "convrot_int8": 1, "asym_w4a8": 1}
L2_FLUSH_BYTES = 256 << 20
INT8_PER_BF16 = 2.0  # nominal dense int8 : bf16 tensor throughput (4.5 : 2.25 PFLOP/s)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="edit20b", choices=sorted(WORKLOAD_DESC))
    ap.add_argument("--no-small-m", action="store_true", help="leave out the M <= 16 HBM record")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default=None, help="restrict the workload to the linear with this name")
    ap.add_argument("--no-graph", action="store_true", help="launch the step eagerly instead of replaying a CUDA graph")
    ap.add_argument("--group", type=int, default=256, choices=[256, 64, 16],
                    help="ConvRot rotation group of the W4A4 linears (the convrot_groupsize variants)")
    ap.add_argument("--flush", choices=["write+read", "write"], default="write+read",
                    help="L2 flush between timed steps: a 256 MiB write, then (default) a 256 MiB read of a "
                         "second buffer so that the write-back of the dirty lines is not charged to the step")
    return ap.parse_args()


def job_time_ms(local_ms, world, dist, torch, device):
    """The job's time: the maximum over ranks of each rank's device time
    (every rank runs a full replica of the step)."""
    if world <= 1:
        return local_ms
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tops(ops_per_step, steps, job_ms, world):
    """Whole-job throughput: the work of all ranks' replicas over the job time."""
    return max(world, 1) * ops_per_step * steps / (job_ms * 1e-3) / 1e12


def step_ops(shapes):
    return sum(2.0 * s.M * s.N * s.K for s in shapes)


def weight_bytes(s):
    """Bytes of the stored weight codes: 4-bit packed, int8, or 4-bit
    codebook indices plus one e4m3 scale per 16 and the 16-level codebook."""
    if s.fmt == "asym_w4a8":
        return s.N * s.K // 2 + s.N * s.K // 16 + 64
    return s.N * s.K // 2 if s.fmt == "w4a4" else s.N * s.K


def alg_bytes(s):
    """Algorithmic HBM bytes of one fused linear: x, W codes, s_w, bias, y."""
    return 2 * s.M * s.K + weight_bytes(s) + 4 * s.N + 2 * s.N + 2 * s.M * s.N


def gemm_alg_bytes(s):
    """Algorithmic bytes of the GEMM launch: W codes, activation codes as bytes,
    scales, bias, y."""
    return weight_bytes(s) + s.M * s.K + 4 * s.M + 6 * s.N + 2 * s.M * s.N


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def make_flusher(torch, dev, mode):
    """L2 flush between timed steps.  A write of a buffer larger than L2 evicts
    every input; with mode "write+read" a read of a second such buffer then
    replaces the (dirty) written lines with clean ones, so that their
    write-back to HBM is not charged to the next timed step."""
    wbuf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    rbuf = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev) if mode == "write+read" else None

    def flush():
        wbuf.zero_()
        if rbuf is not None:
            torch.amax(rbuf)

    return flush


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and throttle reasons while the timed steps run, from two
    readers: `nvidia-smi` every 200 ms (the fields of the usual clocks line)
    and, where the NVML library answers, a thread that reads the same
    values every 2 ms, so that a timed region of a few ms still gets samples
    from inside it.  Both only read; NVML failures leave the nvidia-smi
    record alone."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, torch_device: int):
        self.torch_device = torch_device
        self.gpu = torch_device  # NVML / nvidia-smi index; resolved by PCI location where NVML answers
        self.proc = None
        self.path = None
        self.nvml_thread = None
        self.nvml_stop = None
        self.nvml_samples = []   # (sm MHz, max MHz, reason names)

    def _nvml_loop(self, nvml, handle, bits):
        try:
            smax = float(nvml.nvmlDeviceGetMaxClockInfo(handle, nvml.NVML_CLOCK_SM))
            while not self.nvml_stop.is_set():
                sm = float(nvml.nvmlDeviceGetClockInfo(handle, nvml.NVML_CLOCK_SM))
                active = nvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.nvml_samples.append((sm, smax, [n for n, b in bits if active & b]))
                self.nvml_stop.wait(0.002)
        except Exception:  # noqa: BLE001 -- best effort: the nvidia-smi record stands
            pass

    def _resolve_index(self, nvml):
        """The NVML index of the torch device (its PCI domain, bus and device),
        which differs from the CUDA ordinal when CUDA_VISIBLE_DEVICES is set."""
        import torch
        props = torch.cuda.get_device_properties(self.torch_device)
        want = (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
        for i in range(nvml.nvmlDeviceGetCount()):
            pi = nvml.nvmlDeviceGetPciInfo(nvml.nvmlDeviceGetHandleByIndex(i))
            if (pi.domain, pi.bus, pi.device) == want:
                return i
        return None

    def _start_nvml(self):
        try:
            import threading
            import pynvml as nvml
            handle = nvml.nvmlDeviceGetHandleByIndex(self.gpu)
            bits = [("hw_slowdown", nvml.nvmlClocksEventReasonHwSlowdown),
                    ("hw_thermal_slowdown", nvml.nvmlClocksEventReasonHwThermalSlowdown),
                    ("sw_thermal_slowdown", nvml.nvmlClocksEventReasonSwThermalSlowdown),
                    ("sw_power_cap", nvml.nvmlClocksEventReasonSwPowerCap)]
            self.nvml_stop = threading.Event()
            self.nvml_thread = threading.Thread(target=self._nvml_loop, args=(nvml, handle, bits), daemon=True)
            self.nvml_thread.start()
        except Exception:  # noqa: BLE001 -- no NVML here: nvidia-smi only
            self.nvml_thread = None

    def _stop_nvml(self):
        if self.nvml_thread is not None:
            self.nvml_stop.set()
            self.nvml_thread.join(timeout=2.0)
        if not getattr(self, "nvml_ok", False):
            return
        try:
            import pynvml as nvml
            nvml.nvmlShutdown()
        except Exception:  # noqa: BLE001
            pass

    def start(self):
        try:
            import pynvml as nvml
            nvml.nvmlInit()
            self.nvml_ok = True
            idx = self._resolve_index(nvml)
            if idx is not None:
                self.gpu = idx
        except Exception:  # noqa: BLE001 -- no NVML: the CUDA ordinal, nvidia-smi only
            self.nvml_ok = False
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu)], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        if self.nvml_ok:
            self._start_nvml()

    def stop(self):
        self._stop_nvml()
        sm, smax, reasons = [], None, set()
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 9:
                        continue
                    try:
                        sm.append(float(parts[1]))
                        smax = float(parts[2])
                    except ValueError:
                        continue
                    for n, v in zip(self.REASONS, parts[5:9]):
                        if v.lower().startswith("active"):
                            reasons.add(n)
            os.unlink(self.path)
        out = None
        if sm:
            out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                   "samples": len(sm), "source": "nvidia-smi every 200 ms"}
        if self.nvml_samples:
            nsm = [x[0] for x in self.nvml_samples]
            nreasons = set(r for x in self.nvml_samples for r in x[2])
            nv = {"sm_mhz": statistics.median(nsm), "sm_min_mhz": min(nsm), "sm_max_mhz": self.nvml_samples[0][1],
                  "reasons": sorted(nreasons), "samples": len(nsm),
                  "source": "NVML every 2 ms during the timed steps (the thread runs while the host is free)",
                  "nvml_index": self.gpu}
            if out is None or len(nsm) >= 3:
                # the headline: the samples taken inside the timed steps, with
                # the reasons either reader saw
                smi = out
                out = dict(nv, reasons=sorted(nreasons | set(smi["reasons"] if smi else [])))
                if smi is not None:
                    out["nvidia_smi"] = smi
            else:
                out["reasons"] = sorted(set(out["reasons"]) | nreasons)
                out["nvml"] = nv
        return out


# ------------------------------------------------------------------ the oracle leg

def oracle_inputs(oracle, workload, s):
    """(shape, x, weight codes, weight scales, bias) for the oracle, prepared
    in the linear's format (weight preparation is not timed)."""
    x = synthetic.activations(workload, s.M, s.K, seed_extra=synthetic.source_seed(s.source))
    w, b = synthetic.weights(workload, s.N, s.K, seed_extra=synthetic.source_seed(s.name))
    if s.fmt == "w4a4":
        wq, s_w = oracle.pack_weight(w)
    elif s.fmt == "asym_w4a8":
        idx, s_rel, cb, s_w = synthetic.asym_format(workload, s.N, s.K, seed_extra=synthetic.source_seed(s.name))
        wq = (idx, s_rel, cb)
    else:
        wq, s_w = oracle.quant8(w, *ORACLE_FORMAT[s.fmt])
    return s, x, wq, s_w, b


ORACLE_FORMAT = {"int8_tensorwise": (0, False), "convrot_int8": (256, True)}  # (group, per_row)


def oracle_linear(oracle, s, x, wq, s_w, b):
    if s.fmt == "w4a4":
        return oracle.linear(x, wq, s_w, b, s.K)
    if s.fmt == "asym_w4a8":
        return oracle.asym_linear(x, *wq, s_w, b)
    return oracle.linear8(x, wq, s_w, b, *ORACLE_FORMAT[s.fmt])


def _oracle_rows(oracle, inputs, rows, threads):
    """The oracle on the first ``rows`` rows of every linear, split into
    ``threads`` row ranges run at once (the oracle's C calls release the GIL,
    so each runs on its own core); returns (ops, seconds)."""
    from concurrent.futures import ThreadPoolExecutor
    jobs = []
    for s, x, wq, s_w, b in inputs:
        r = min(rows, s.M)
        cuts = sorted({(r * i) // threads for i in range(threads + 1)})
        jobs += [(s, x[a:c], wq, s_w, b) for a, c in zip(cuts[:-1], cuts[1:]) if c > a]
    ops = sum(2.0 * j[1].shape[0] * j[0].N * j[0].K for j in jobs)
    t0 = time.perf_counter()
    if threads == 1:
        for j in jobs:
            oracle_linear(oracle, *j)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda j: oracle_linear(oracle, *j), jobs))
    return ops, time.perf_counter() - t0


def cpu_baseline(shapes, workload, budget_s=15.0):
    """Time the CPU oracle (as it stands) on a bounded sample: the first ``r``
    rows of each linear of the step, r grown until one thread takes about
    ``budget_s``; throughput in the metric's unit (TOPS).  The same sample is
    then run again split over every core of the host (``all_cores``)."""
    import oracle
    inputs = [oracle_inputs(oracle, workload, s) for s in shapes]
    rows = 1
    while True:
        ops, dt = _oracle_rows(oracle, inputs, rows, 1)
        if dt >= budget_s / 3 or rows >= max(s.M for s in shapes):
            break
        rows = min(max(s.M for s in shapes), rows * max(2, int(budget_s / 3 / max(dt, 1e-3))))
    ncpu = os.cpu_count() or 1
    ops_all, dt_all = _oracle_rows(oracle, inputs, rows, ncpu)
    sample = (f"first {rows} rows (capped at M) of each of the {len(shapes)} linears of one step "
              f"({ops / 1e9:.2f} GOP); weight packing untimed")
    return {"value": ops / dt / 1e12, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": sample + f"; {dt:.1f} s on one thread",
            "seconds": dt, "host": host_cpu(),
            "all_cores": {"value": ops_all / dt_all / 1e12, "unit": UNIT, "cores": ncpu, "kind": "oracle",
                          "sample": sample + f", split into {ncpu} row ranges run at once: {dt_all:.2f} s",
                          "seconds": dt_all}}


def host_cpu():
    """The host the oracle ran on: logical CPUs and the CPU model name."""
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"logical_cpus": os.cpu_count(), "model": model}


# ------------------------------------------------------------------ main

def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    shapes = synthetic.workload_shapes(args.workload)
    if args.only:
        shapes = [s for s in shapes if s.name == args.only]
        if not shapes:
            raise SystemExit(f"no linear named {args.only!r} in workload {args.workload}")
    config = {"workload": args.workload, "description": WORKLOAD_DESC[args.workload], "convrot_group": args.group,
              "linears": [f"{s.name}:M{s.M}xK{s.K}xN{s.N}" for s in shapes],
              "l2": ("flushed between timed steps, outside the events: 256 MiB write, then 256 MiB read of a second "
                     "buffer (inputs cold, no dirty lines left in L2)") if args.flush == "write+read"
                    else "flushed between timed steps, outside the events: 256 MiB write",
              "launch": ("each step replayed from a CUDA graph" if not args.no_graph else "eager launches")
                        + ": per input tensor one rotate+quantize launch, then one GEMM launch per linear reading it",
              "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
              "codes": "s4 packed weights, s4 activations widened to s8 for tcgen05 kind::i8, int32 accumulate, "
                       "fp32 epilogue, bf16 out"}

    if args.impl == "reference":
        return reference_arm(args, shapes, config, world, rank)

    import torch
    import torch.distributed as dist
    import rotation_quantized_bit_b200 as rq

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    rq.load_library()
    # Dense int8 tensor-core rate of this GPU from the library's own no-memory
    # tcgen05.mma.kind::i8 loop (128 x 256 x 32, all SMs), reported beside the
    # roofline; the roofline's peak itself is the measured bf16 rate x 2.
    mma_i8_tops, _ = rq.convrot_measure_mma_i8(256, False, 4096)

    # ---- inputs (untimed): one activation tensor per source (linears of a
    # layer that read the same tensor share it), packed weights per linear
    xs = {}
    for s in shapes:
        if s.source not in xs:
            xb = synthetic.activations(args.workload, s.M, s.K, seed_extra=synthetic.source_seed(s.source))
            xs[s.source] = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
    layers = []
    for s in shapes:
        w, b = synthetic.weights(args.workload, s.N, s.K, seed_extra=synthetic.source_seed(s.name))
        wd = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).to(dev)
        if s.fmt == "w4a4":
            wq, s_w = rq.convrot_pack_weight_g(wd, args.group)
        elif s.fmt == "asym_w4a8":
            # weights arrive converted offline (no bf16 -> codebook conversion
            # runs here): seeded tensors in the storage layout
            idx, s_rel, cb, sch = synthetic.asym_format(args.workload, s.N, s.K,
                                                        seed_extra=synthetic.source_seed(s.name))
            wq = tuple(torch.from_numpy(a).to(dev) for a in (idx, s_rel, cb))
            s_w = torch.from_numpy(sch).to(dev)
        else:
            wq, s_w = rq.w8a8_pack_weight(wd, FORMAT_ID[s.fmt])
        bias = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)
        y = torch.empty((s.M, s.N), dtype=torch.bfloat16, device=dev)
        layers.append((s, wq, s_w, bias, y))
        del wd
    # groups of linears that read one source, in order of first use
    groups = []
    for i, (s, *_r) in enumerate(layers):
        for g in groups:
            if g[0] == s.source:
                g[1].append(i)
                break
        else:
            groups.append((s.source, [i]))
    ws_bytes = max(rq.convrot_w4a4_workspace_size(s.M, s.N, s.K) if s.fmt == "w4a4"
                   else rq.asym_w4a8_workspace_size(s.M, s.N, s.K) if s.fmt == "asym_w4a8"
                   else rq.w8a8_workspace_size(s.M, s.N, s.K, FORMAT_ID[s.fmt]) for s in shapes)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    # int8 formats: the activation codes and scales of each source
    q8 = {}
    for s in shapes:
        if s.fmt != "w4a4" and s.source not in q8:
            q8[s.source] = (torch.empty((s.M, s.K), dtype=torch.int8, device=dev),
                            torch.empty((s.M if FORMAT_ID[s.fmt] == 1 else 1,), dtype=torch.float32, device=dev))
    flush = make_flusher(torch, dev, args.flush)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()

    nlin = len(layers)
    ngrp = len(groups)

    def run_step(evs=None, per_kernel=False):
        """One step: per source, one rotate + quantize, then the GEMM of every
        linear that reads it.  evs[g] = [start, after quantize, after each
        GEMM]; in the timed step only the group's start and end are recorded
        (so the GEMMs' programmatic launches overlap what precedes them), in
        the per-kernel breakdown every boundary is."""
        cur = torch.cuda.current_stream()  # the capture stream while a graph is being captured
        for gi, (src, idx) in enumerate(groups):
            ev = evs[gi] if evs is not None else None
            if ev is not None:
                ev[0].record(cur)
            fmt = layers[idx[0]][0].fmt
            if fmt == "w4a4":
                rq.convrot_w4a4_quantize_g(xs[src], ws, args.group)
            else:
                rq.w8a8_quantize(xs[src], FORMAT_ID[fmt], x8=q8[src][0], s_x=q8[src][1], workspace=ws)
            if ev is not None and per_kernel:
                ev[1].record(cur)
            for j, i in enumerate(idx):
                s, wq, s_w, bias, y = layers[i]
                if fmt == "w4a4":
                    rq.convrot_w4a4_gemm_quantized(ws, s.M, wq, s_w, bias, out=y)
                elif fmt == "asym_w4a8":
                    rq.asym_w4a8_gemm(q8[src][0], q8[src][1], *wq, s_w, bias, out=y)
                else:
                    rq.w8a8_gemm(q8[src][0], q8[src][1], wq, s_w, bias, FORMAT_ID[fmt], out=y)
                if ev is not None and (per_kernel or j == len(idx) - 1):
                    ev[2 + j].record(cur)

    for _ in range(max(args.warmup, 3)):
        flush()
        run_step()
    torch.cuda.synchronize()

    # One CUDA graph per timed step (each with its own events); a replay runs
    # the step's launches back to back, with no host gaps.  External events:
    # recorded inside a capture they become event-record nodes timestamped on
    # every replay.
    def make_events():
        return [[[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 + len(idx))]
                 for (_src, idx) in groups] for _ in range(args.steps)]

    step_events, kern_events = make_events(), make_events()
    graphs, kgraphs = [], []
    if not args.no_graph:
        for k in range(args.steps):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                run_step(step_events[k])
            graphs.append(g)
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2):
                run_step(kern_events[k], per_kernel=True)
            kgraphs.append(g2)
        for g in (graphs[0], kgraphs[0]):  # one untimed replay of each
            flush()
            g.replay()
        torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    counts0 = rq.convrot_dispatch_counts()
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 or world == 1 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    for k in range(args.steps):
        flush()  # L2 flush, outside the step's events
        if graphs:
            graphs[k].replay()
        else:
            run_step(step_events[k])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    counts1 = rq.convrot_dispatch_counts()
    # Per-kernel breakdown (for the roofline of the dominant kernel): the same
    # step with an event between every two launches.
    for k in range(args.steps):
        flush()
        if kgraphs:
            kgraphs[k].replay()
        else:
            run_step(kern_events[k], per_kernel=True)
    torch.cuda.synchronize()
    err = rq.convrot_device_error()
    if err:
        raise RuntimeError(f"device error word {err:#x}: a bounded wait expired")
    if graphs:  # launches of a replayed graph are not seen by the host counters
        launches = (ngrp + nlin) * args.steps
    else:
        launches = (counts1["rotate_quant"] - counts0["rotate_quant"]) + (counts1["tc_gemm"] - counts0["tc_gemm"]) + \
                   (counts1["tc_gemm_splitk"] - counts0["tc_gemm_splitk"])

    # per-group times of the timed steps, and per-kernel times of the
    # breakdown steps (ms), summed over the K steps
    t_grp = np.zeros(ngrp)
    t_quant = np.zeros(ngrp)
    t_gemm = np.zeros(nlin)
    step_ms = np.zeros(args.steps)  # this rank's device time of each timed step
    for k in range(args.steps):
        for gi, (_src, idx) in enumerate(groups):
            ev = step_events[k][gi]
            tg = ev[0].elapsed_time(ev[1 + len(idx)])
            t_grp[gi] += tg
            step_ms[k] += tg
            kv = kern_events[k][gi]
            t_quant[gi] += kv[0].elapsed_time(kv[1])
            for j, i in enumerate(idx):
                t_gemm[i] += kv[1 + j].elapsed_time(kv[2 + j])
    total_ms = job_time_ms(float(t_grp.sum()), world, dist, torch, dev)
    ms_per_step = total_ms / args.steps
    ops = step_ops(shapes)
    value = job_tops(ops, args.steps, total_ms, world)

    peaks = load_peaks()
    int8_peak = peaks["bf16_tflops"] * INT8_PER_BF16
    detail = []
    for gi, (src, idx) in enumerate(groups):
        s0 = layers[idx[0]][0]
        tq, tgrp = t_quant[gi] / args.steps, t_grp[gi] / args.steps
        gops = sum(2.0 * layers[i][0].M * layers[i][0].N * layers[i][0].K for i in idx)
        entry = {"input": src, "format": s0.fmt, "M": s0.M, "K": s0.K, "us_group": round(tgrp * 1e3, 2),
                 "tops_group": round(gops / (tgrp * 1e-3) / 1e12, 1), "us_prologue": round(tq * 1e3, 2),
                 "prologue_hbm_gbs": round((3.0 * s0.M * s0.K + 4 * s0.M) / (tq * 1e-3) / 1e9, 1), "linears": []}
        for i in idx:
            s = layers[i][0]
            tg = t_gemm[i] / args.steps
            op = 2.0 * s.M * s.N * s.K
            gemm_bytes = gemm_alg_bytes(s)
            entry["linears"].append({
                "linear": s.name, "N": s.N, "us_gemm": round(tg * 1e3, 2),
                "gemm_tops": round(op / (tg * 1e-3) / 1e12, 1),
                "gemm_frac_int8_peak": round(op / (tg * 1e-3) / 1e12 / int8_peak, 3),
                "gemm_hbm_gbs": round(gemm_bytes / (tg * 1e-3) / 1e9, 1)})
        detail.append(entry)
    # dominant kernel = the single launch with the largest share of the step
    cand = [("gemm", i, t_gemm[i]) for i in range(nlin)] + [("prologue", gi, t_quant[gi]) for gi in range(ngrp)]
    kind, idx, tsum = max(cand, key=lambda c: c[2])
    t_launch = tsum / args.steps * 1e-3  # seconds per launch
    if kind == "gemm":
        s = layers[idx][0]
        ridge = int8_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
        gemm_bytes = gemm_alg_bytes(s)
        intensity = 2.0 * s.M * s.N * s.K / gemm_bytes
        if intensity >= ridge:
            roof = {"bound": "tensor", "achieved": 2.0 * s.M * s.N * s.K / t_launch / 1e12,
                    "peak": int8_peak, "unit": "TFLOP/s"}
        else:
            roof = {"bound": "hbm", "achieved": gemm_bytes / t_launch / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
        kname = "w4a4_tc_gemm_kernel"
        roof["launch"] = f"{s.name} M{s.M} K{s.K} N{s.N}"
    else:
        s = layers[groups[idx][1][0]][0]
        roof = {"bound": "hbm", "achieved": (3.0 * s.M * s.K + 4 * s.M) / t_launch / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s"}
        kname = "rotate_quant_kernel"
        roof["launch"] = f"prologue of {groups[idx][0]} M{s.M} K{s.K}"
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = kname
    roof["peak_source"] = (f"{peaks['source']} bf16 dense burst {peaks['bf16_tflops']} TFLOP/s x {INT8_PER_BF16} "
                           "(nominal int8:bf16)" if roof["bound"] == "tensor" else f"{peaks['source']} HBM copy")
    roof["share_of_breakdown"] = float(tsum / (t_quant.sum() + t_gemm.sum()))
    if roof["bound"] == "tensor":
        roof["int8_mma_measured_tops"] = round(mma_i8_tops, 1)
        roof["frac_of_int8_mma_measured"] = roof["achieved"] / mma_i8_tops
    roof["traffic"] = committed_traffic(kname, s)
    roof["timing"] = ("average launch duration from a second graph of the same step with an event between every "
                      "two launches (this serialises the programmatic-launch overlap of the timed step)")

    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(args, rq, torch, dev, stream, shapes, xs, layers, groups, ws, flush, world, dist)

    small = None
    if rank == 0 and not args.no_small_m:
        small = small_m_record(rq, torch, dev, flush, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(shapes, args.workload)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": max(world, 1), "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": round(ms_per_step, 4),
        "step_ms_percentiles": {"p10": round(float(np.percentile(step_ms, 10)), 4),
                                "median": round(float(np.median(step_ms)), 4),
                                "p90": round(float(np.percentile(step_ms, 90)), 4), "rank": rank},
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic",
        "config": config, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
        "clocks": clocks, "small_m": small, "detail": detail,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs, kgraphs
    if world > 1:
        dist.destroy_process_group()


def committed_traffic(kernel, s):
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.json),
    if it was taken on this launch shape and on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            rec = json.load(f)
        ents = rec.get(kernel) or []
        if isinstance(ents, dict):
            ents = [ents]
        sha = source_sha(kernel)
        for ent in ents:
            if ent.get("source_sha256") == sha and ent.get("shape") == [s.M, s.K, s.N]:
                return ent["dram_bytes_per_launch"]
        return None
    except (OSError, ValueError, KeyError):
        return None


def source_sha(kernel):
    fname = {"w4a4_tc_gemm_kernel": "gemm.cu", "rotate_quant_kernel": "rotate_quant.cu"}[kernel]
    with open(os.path.join(ROOT, "rotation_quantized_bit_b200", "csrc", fname), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


SMALL_M_SHAPES = [(2560, 9728), (9728, 2560), (3072, 12288), (12288, 3072)]  # (K, N) of the small-M sweep
SMALL_M_TOKENS = [1, 8, 16]


def small_m_record(rq, torch, dev, flush, peaks, reps=5):
    """HBM GB/s of the fused Linear (rotate+quantize, then the GEMM) and of the
    GEMM alone at M in {1, 8, 16} over the small-M sweep's (K, N) shapes.

    Each figure is a steady-state per-call time: R back-to-back calls in one
    CUDA graph, each on its own copy of the packed weights (R copies hold more
    than three times the L2), L2 flushed before every replay, the median of
    ``reps`` replays divided by R.  Bytes are the algorithmic ones: for the
    Linear x (2MK) + weights (NK/2) + s_w, bias (6N) + y (2MN); for the GEMM
    the packed codes and scales (MK/2 + 4M) instead of x.  The GEMM calls
    share one quantization, as projections that read one tensor do."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    out = []
    for K, N in SMALL_M_SHAPES:
        w, b = synthetic.weights("small_m", N, K)
        wd = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).to(dev)
        wq0, s_w = rq.convrot_pack_weight(wd)
        del wd
        bias = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)
        R = max(8, int(np.ceil(3.0 * l2 / wq0.numel())))
        wqs = [wq0] + [wq0.clone() for _ in range(R - 1)]
        for M in SMALL_M_TOKENS:
            x = torch.from_numpy(synthetic.activations("small_m", M, K).view(np.int16)).view(torch.bfloat16).to(dev)
            ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(R)]
            ws = torch.empty(rq.convrot_w4a4_workspace_size(M, N, K), dtype=torch.uint8, device=dev)
            rq.convrot_w4a4_quantize(x, ws)

            def ring_gemm():
                for r in range(R):
                    rq.convrot_w4a4_gemm_quantized(ws, M, wqs[r], s_w, bias, out=ys[r])

            def ring_linear():
                for r in range(R):
                    rq.convrot_w4a4_linear(x, wqs[r], s_w, bias, out=ys[r], workspace=ws)

            rec = {"M": M, "K": K, "N": N, "calls_per_replay": R}
            for name, fn, nbytes in (
                    ("gemm", ring_gemm, N * K / 2 + 6 * N + M * K / 2 + 4 * M + 2 * M * N),
                    ("linear", ring_linear, 2 * M * K + N * K / 2 + 6 * N + 2 * M * N)):
                side = torch.cuda.Stream()
                side.wait_stream(torch.cuda.current_stream())
                with torch.cuda.stream(side):
                    fn()  # warm-up outside the capture
                torch.cuda.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    fn()
                times = []
                for _ in range(reps):
                    flush()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    g.replay()
                    e1.record()
                    e1.synchronize()
                    times.append(e0.elapsed_time(e1))
                us = statistics.median(times) * 1e3 / R
                gbs = nbytes / (us * 1e-6) / 1e9
                rec[f"{name}_us"] = round(us, 2)
                rec[f"{name}_gbs"] = round(gbs, 1)
                rec[f"{name}_frac_hbm"] = round(gbs / peaks["hbm_gbs"], 3)
                del g
            out.append(rec)
            del ys, ws, x
        del wqs, wq0
        torch.cuda.empty_cache()
    if rq.convrot_device_error():
        raise RuntimeError("device error word set during the small-M record")
    fr_l = [r["linear_frac_hbm"] for r in out]
    fr_g = [r["gemm_frac_hbm"] for r in out]
    return {"peak_gbs": peaks["hbm_gbs"], "peak_source": f"{peaks['source']} HBM copy",
            "linear_frac_hbm": {"min": min(fr_l), "median": statistics.median(fr_l), "max": max(fr_l)},
            "gemm_frac_hbm": {"min": min(fr_g), "median": statistics.median(fr_g), "max": max(fr_g)},
            "method": "back-to-back calls in one CUDA graph over distinct weight copies (> 3x L2), L2 flushed "
                      "before each replay; per-call time = median replay time / calls",
            "kernels": "M <= 16: one-CTA-per-token prologue (rq_rows_kernel) + bandwidth-bound slab GEMM "
                       "(w4a4_gemv_kernel: bulk-copied weight rows, mma.sync s8)",
            "shapes": out}


def end_to_end(args, rq, torch, dev, stream, shapes, xs, layers, groups, ws, flush, world, dist):
    """Same step through the public C-ABI calls (convrot_w4a4_quantize once per
    source, convrot_w4a4_gemm_quantized per linear; convrot_w4a4_linear when a
    source feeds one linear), with the step's inputs copied from pinned host
    memory and every output read back, inside the timing.  The copies run on
    two copy streams, pipelined per input group: a group's input is copied in
    while the previous groups compute, and its outputs are copied out while
    the next groups compute."""
    host_x = {k: v.cpu().pin_memory() for k, v in xs.items()}
    host_y = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for (_, _, _, _, y) in layers]
    h2d = sum(v.numel() * 2 for v in host_x.values())
    d2h = sum(y.numel() * 2 for y in host_y)
    c_in, c_out = torch.cuda.Stream(), torch.cuda.Stream()

    def run_group(src, idx):
        fmt = layers[idx[0]][0].fmt
        if len(idx) == 1:
            s, wq, s_w, bias, y = layers[idx[0]]
            if fmt == "w4a4":
                rq.convrot_w4a4_linear_g(xs[src], wq, s_w, bias, args.group, out=y, workspace=ws)
            elif fmt == "asym_w4a8":
                rq.asym_w4a8_linear(xs[src], *wq, s_w, bias, out=y, workspace=ws)
            else:
                rq.w8a8_linear(xs[src], wq, s_w, bias, FORMAT_ID[fmt], out=y, workspace=ws)
            return
        if fmt == "w4a4":
            rq.convrot_w4a4_quantize_g(xs[src], ws, args.group)
        else:
            x8, sx = rq.w8a8_quantize(xs[src], FORMAT_ID[fmt], workspace=ws)
        for i in idx:
            s, wq, s_w, bias, y = layers[i]
            if fmt == "w4a4":
                rq.convrot_w4a4_gemm_quantized(ws, s.M, wq, s_w, bias, out=y)
            elif fmt == "asym_w4a8":
                rq.asym_w4a8_gemm(x8, sx, *wq, s_w, bias, out=y)
            else:
                rq.w8a8_gemm(x8, sx, wq, s_w, bias, FORMAT_ID[fmt], out=y)

    def step():
        comp = torch.cuda.current_stream()
        c_in.wait_stream(comp)   # the previous step is done with the device inputs
        c_out.wait_stream(comp)
        ev_in = []
        with torch.cuda.stream(c_in):
            for src, _idx in groups:
                xs[src].copy_(host_x[src], non_blocking=True)
                e = torch.cuda.Event()
                e.record(c_in)
                ev_in.append(e)
        for gi, (src, idx) in enumerate(groups):
            comp.wait_event(ev_in[gi])
            run_group(src, idx)
            done = torch.cuda.Event()
            done.record(comp)
            c_out.wait_event(done)
            with torch.cuda.stream(c_out):
                for i in idx:
                    host_y[i].copy_(layers[i][4], non_blocking=True)
        comp.wait_stream(c_out)  # the step ends when its last output is on the host

    for _ in range(max(args.warmup, 3)):
        flush()
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total = 0.0
    for _ in range(args.steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        e1.synchronize()
        total += e0.elapsed_time(e1)
    total = job_time_ms(total, world, dist, torch, dev)
    return {"value": round(job_tops(step_ops(shapes), args.steps, total, world), 2), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(total / args.steps, 4),
            "api": "C ABI: convrot_w4a4_quantize_g per source + convrot_w4a4_gemm_quantized per linear "
                   "(convrot_w4a4_linear_g for single-linear sources; w8a8_* for the int8 formats); "
                   "pinned host->device x and device->host y on two copy streams, pipelined per input group"}


def reference_arm(args, shapes, config, world, rank):
    """The CPU oracle as the reference arm: rank 0 only, bounded sample per step."""
    if rank != 0:
        return
    import oracle
    inputs = [oracle_inputs(oracle, args.workload, s) for s in shapes]
    rows = 2  # rows per linear per step: keeps a step near a few seconds

    def step():
        ops = 0.0
        for s, x, wq, s_w, b in inputs:
            r = min(rows, s.M)
            oracle_linear(oracle, s, x[:r], wq, s_w, b)
            ops += 2.0 * r * s.N * s.K
        return ops

    for _ in range(max(args.warmup, 3) if args.warmup else 0):
        step()
    t0 = time.perf_counter()
    ops = 0.0
    for _ in range(args.steps):
        ops += step()
    dt = time.perf_counter() - t0
    value = ops / dt / 1e12
    sample = f"first {rows} rows of each of the {len(shapes)} linears per step ({ops / args.steps / 1e9:.2f} GOP/step)"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": max(world, 1), "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32/int64", "data": "synthetic", "config": config,
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
                             "host": host_cpu()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _rank_entry(rank, world, port):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    main()


def self_launch(n):
    """``--gpus N`` without torchrun: start the N ranks here (one process per
    GPU, spawned), each running main() with the environment torchrun sets."""
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    mp.start_processes(_rank_entry, args=(n, port), nprocs=n, start_method="spawn", join=True)


if __name__ == "__main__":
    _args = parse()
    if _args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        self_launch(_args.gpus)
    else:
        main()
