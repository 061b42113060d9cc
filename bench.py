#!/usr/bin/env python
"""Benchmark of the B200 WKV forward / diagonal scan library.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step is one pass of the hot path over one batch of synthetic input
already resident in HBM: a WKV forward (or, for ``--workload scan_mingru``,
a diagonal scan).  The default workload is the largest single-GPU WKV
forward: the long-sequence one (fp32, B=1, T=131072, C=1024, keys of
standard deviation 3, slow decays); ``--workload`` selects the others.  W untimed warm-up steps and a short untimed soak
run first; then exactly K steps are timed with CUDA events on the launching
stream, bracketed by a barrier and a device synchronisation, and the maximum
over ranks is taken.  Inputs rotate over enough buffer sets that the data a
step touches is not in L2 from the step before (each set is re-read only
after >= 3x the L2 size of other traffic).

Printed (rank 0): one JSON line with the metric, the roofline of the kernel
(algorithmic bytes / average CUDA-event launch duration against the measured
HBM peak), the float64 CPU oracle timed on this host's cores, an end-to-end
number through the C ABI with host buffers (host->device copies, the call,
device->host copy of the result, every step), SM clocks sampled during the
timed region (NVML queries every fraction of a millisecond while the timed
steps run; null when none landed inside it), and the number of library
kernel launches timed.  The CPU oracle is timed on all of this host's cores
and on one core.

``--shape B,T,C`` runs a workload's distributions at another shape (the
same kernel on a smaller case, for profiler captures); the JSON line's
config says so.

``--impl reference`` times the CPU oracle instead (the only reference this
project has: a plain float64 implementation of the pages' definition), on a
bounded sample of the same workload, and prints the same line with
"impl": "reference".  Multi-GPU runs (torchrun) give every rank its own copy
of the workload (weak scaling, no collective in the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "WKV fwd B·T·C elems/s and achieved HBM GB/s vs B200 peak (1 GPU)"
FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "rwkv_wkv_mixing_b200", "csrc")


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--workload", default="wkv_long", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--soak-seconds", type=float, default=1.0,
                    help="untimed steps before the timed region, so clocks settle")
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="budget of each CPU-oracle leg, all cores and one core (rank 0, N=1)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--tile-steps", type=int, default=0,
                    help="steps per tile (8, 32, 64, 128, 256); 0 keeps the library default")
    ap.add_argument("--launch", default="graph", choices=["graph", "direct"],
                    help="replay the K steps from CUDA graphs (default) or call directly")
    ap.add_argument("--shape", default=None,
                    help="B,T,C (B,T,D for scans): the workload's distributions at another "
                         "shape, for small profiler captures of the same kernel")
    return ap.parse_args(argv)


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the sources every kernel is built from (their dispatch included); a
# recorded DRAM-traffic figure is only reported while these are unchanged
KERNEL_SOURCES = ("capi.cu", "capi_backward.cuh", "capi_host.cuh", "persistent_scan.cuh",
                  "persistent_wkv.cuh", "persistent_bwd.cuh", "chunked_scan.cuh", "scan_common.cuh",
                  "wkv_ops.cuh", "lru_ops.cuh", "wkv_backward.cuh", "serial_wkv.cuh",
                  "token_shift.cuh", "ptx.cuh")


def _code_only(text):
    """C/C++ source without comments and with whitespace collapsed, so that
    an edit of comments alone does not count as a change of the kernels."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif c in "\"'":  # string or character literal, kept whole
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


# The gradients' own sources (kernels and host side): no forward kernel is
# built from them.  The host-buffer pipeline: no device kernel is.
GRAD_ONLY_SOURCES = ("capi_backward.cuh", "persistent_bwd.cuh", "wkv_backward.cuh")
HOST_ONLY_SOURCES = ("capi_host.cuh",)
FORWARD_SOURCES = tuple(n for n in KERNEL_SOURCES
                        if n not in GRAD_ONLY_SOURCES and n not in HOST_ONLY_SOURCES)
GRAD_SOURCES = tuple(n for n in KERNEL_SOURCES if n not in HOST_ONLY_SOURCES)


def src_hash(read=None, names=KERNEL_SOURCES):
    """Hash of the code of the named kernel sources (default: every one;
    comments and whitespace ignored); `read(name)` returns a source's text
    (default: the file)."""
    h = hashlib.sha256()
    for name in names:
        if read is None:
            with open(os.path.join(CSRC, name), encoding="utf-8") as f:
                text = f.read()
        else:
            text = read(name)
        h.update(name.encode() + b"\0" + _code_only(text).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per launch from a committed ncu capture, if it was taken on
    the kernel sources as they are now (those the entry names, every kernel
    source when it names none); otherwise None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(workload)
    except Exception:
        return None
    if not rec:
        return None
    names = tuple(rec.get("sources") or KERNEL_SOURCES)
    if not set(names) <= set(KERNEL_SOURCES) or rec.get("src_sha") != src_hash(names=names):
        return None
    return rec.get("dram_bytes_per_launch")


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons, read-only, sampled from a
    background thread: NVML queries every `fast_s` seconds while `fast()` is
    on (around the timed region, so even a few milliseconds of timed steps
    get samples), every 100 ms otherwise; `nvidia-smi -lms 100` when NVML
    cannot be loaded.  Nothing is ever set."""
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid=None, fast_s=0.0002):
        self.samples = []          # (time, sm_mhz, sm_max_mhz, [reason names])
        self.proc = None
        self.source = None
        self._fast = False
        self._stop = False
        self._wake = threading.Event()   # set to cut a slow-mode sleep short
        self._took = threading.Event()   # set by the poller after each sample
        self.fast_s = fast_s
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            h = None
            if gpu_uuid:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(gpu_uuid)
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.nvml, self.handle = pynvml, h
            self.bits = (pynvml.nvmlClocksEventReasonHwSlowdown,
                         pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                         pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                         pynvml.nvmlClocksEventReasonSwPowerCap)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.source = "nvml"
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.nvml = None
        cmd = ["nvidia-smi", f"--query-gpu={self.SMI_FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if gpu_uuid:
            cmd += ["-i", gpu_uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
            return
        self.source = "nvidia-smi"
        self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()

    def _poll_nvml(self):
        nv, h = self.nvml, self.handle
        try:
            reasons_fn = nv.nvmlDeviceGetCurrentClocksEventReasons
        except AttributeError:
            reasons_fn = nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop:
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = int(reasons_fn(h))
                self.samples.append((time.time(), sm, self.max_mhz,
                                     [n for n, b in zip(self.NAMES, self.bits) if r & b]))
            except Exception:
                pass
            self._took.set()
            if self._fast:
                time.sleep(self.fast_s)
            else:
                self._wake.wait(0.1)
                self._wake.clear()

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm, smax = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            self.samples.append((time.time(), sm, smax,
                                 [n for n, r in zip(self.NAMES, parts[4:8])
                                  if r.lower().startswith("active")]))

    def fast(self, on):
        """Switch to (or from) sampling every `fast_s`; switching on returns
        once the poller has taken a sample in fast mode."""
        self._fast = bool(on)
        if on and self.source == "nvml":
            self._took.clear()
            self._wake.set()
            self._took.wait(1.0)

    def stop(self):
        self._stop = True
        self._wake.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.nvml is not None:
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self, t0, t1, timed_ms=None):
        """Samples taken inside [t0, t1] only; sm_mhz is null when none
        landed there.  `mhz_x_ms` is the timed milliseconds times the median
        SM clock, to compare runs at different clocks."""
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": len(win),
               "window": "timed", "source": self.source}
        if not win:
            return out
        med = statistics.median(s[1] for s in win)
        out.update({"sm_mhz": med, "sm_min_mhz": min(s[1] for s in win),
                    "sm_max_mhz": max(s[2] for s in win),
                    "reasons": sorted({n for s in win for n in s[3]})})
        if timed_ms is not None:
            out["mhz_x_ms"] = med * timed_ms
        return out


# ---------------------------------------------------------------------------
# workloads on the device
# ---------------------------------------------------------------------------
class DeviceWorkload:
    """Inputs resident in HBM, rotated over `n_sets` copies, and the C-ABI
    call of one step with raw device pointers.

    kinds: "wkv" (plain, with a state read and written in place, or with the
    receptance gate), "scan" (diagonal scan), "shift" (token shift, the
    saved last token read and written in place)."""

    def __init__(self, name, torch, lib, l2_bytes, shape=None):
        self.name = name
        sB, sT, sC = shape if shape is not None else (None, None, None)
        self.spec = spec = workloads.WORKLOADS[name]
        self.torch = torch
        self.lib = lib
        dev = torch.device("cuda", torch.cuda.current_device())
        self.dev = dev
        self.consts = {}
        self.has_state = self.gated = False
        if isinstance(spec, workloads.ScanSpec):
            self.kind = "scan"
            x = workloads.make_scan(name, B=sB, T=sT, D=sC)
            B, T, C = x.a.shape
            bf = spec.dtype == "bf16"
            self.dtype, self.es = spec.dtype, 2 if bf else 4
            self.host = {"a": x.a_bits.view(np.int16) if bf else x.a,
                         "b": x.b_bits.view(np.int16) if bf else x.b}
            self.outputs = {"h": (B, T, C)}
            alg = 3 * self.es * B * T * C
        elif isinstance(spec, workloads.LruSpec):
            self.kind = "lru"
            x = workloads.make_lru(name, B=sB, T=sT, D=sC)
            B, T, C = x.u.shape[:3]
            self.dtype, self.es = "c64", 8
            self.host = {"u": x.u}
            for k in ("nu_log", "theta_log", "gamma"):
                self.consts[k] = torch.from_numpy(getattr(x, k)).to(dev)
            self.outputs = {"x": (B, T, C, 2)}
            alg = 16 * B * T * C + 12 * C
        elif isinstance(spec, workloads.ShiftSpec):
            self.kind = "shift"
            x = workloads.make_token_shift(name, B=sB, T=sT, C=sC)
            B, T, C = x.x.shape
            bf = spec.dtype == "bf16"
            self.dtype, self.es = spec.dtype, 2 if bf else 4
            self.host = {"x": x.x_bits.view(np.int16) if bf else x.x,
                         "xp": x.x_prev_bits.view(np.int16) if bf else x.x_prev}
            self.consts["mu"] = torch.from_numpy(x.mu).to(dev)
            self.n_mix = x.mu.shape[0]
            self.outputs = {"out": (self.n_mix, B, T, C)}
            alg = self.es * B * T * C * (1 + self.n_mix) + 2 * self.es * B * C + 4 * self.n_mix * C
        else:
            self.kind = "wkv"
            x = workloads.make_wkv(name, B=sB, T=sT, C=sC)
            B, T, C = x.k.shape
            bf = spec.dtype == "bf16"
            self.dtype, self.es = spec.dtype, 2 if bf else 4
            self.host = {"k": x.k_bits.view(np.int16) if bf else x.k,
                         "v": x.v_bits.view(np.int16) if bf else x.v}
            self.gated = x.r is not None
            if self.gated:
                self.host["r"] = x.r_bits.view(np.int16) if bf else x.r
            self.has_state = x.s_in is not None
            if self.has_state:
                self.host["s"] = x.s_in
            self.consts["w"] = torch.from_numpy(x.w).to(dev)
            self.consts["u"] = torch.from_numpy(x.u).to(dev)
            self.outputs = {"y": (B, T, C)}
            alg = self.es * B * T * C * (4 if self.gated else 3) + 8 * C + \
                (24 * B * C if self.has_state else 0)
            if x.gy is not None:   # gradients: read k, v, gy; write gk, gv (and gw, gu)
                self.kind = "bwd"
                self.host["gy"] = x.gy
                self.outputs = {"gk": (B, T, C), "gv": (B, T, C), "gw": (C,), "gu": (C,)}
                alg = 20 * B * T * C + 16 * C
        self.inputs = x
        self.B, self.T, self.C = B, T, C
        self.elements = B * T * C
        self.alg_bytes = alg
        # bytes one step touches, for sizing the rotation against L2
        self.set_bytes = alg
        self.n_sets = 1 if alg >= 3 * l2_bytes else int(np.ceil(3 * l2_bytes / alg)) + 1
        first = {k: self._to_dev(v) for k, v in self.host.items()}
        self.sets = []
        for i in range(self.n_sets):
            st = {k: (t if i == 0 else t.clone()) for k, t in first.items()}
            for k, shape in self.outputs.items():
                st[k] = torch.empty(shape, dtype=first[next(iter(first))].dtype, device=dev)
            self.sets.append(st)
        self.stream = torch.cuda.current_stream()

    def _to_dev(self, arr):
        t = self.torch.from_numpy(np.ascontiguousarray(arr))
        if arr.dtype == np.int16:
            t = t.view(self.torch.bfloat16)
        return t.to(self.dev)

    def api(self):
        if self.kind == "bwd":
            return "wkv_backward"
        if self.kind == "lru":
            return "lru_scan"
        if self.kind == "scan":
            return "diag_scan_bf16" if self.dtype == "bf16" else "diag_scan"
        bf = "_bf16" if self.dtype == "bf16" else ""
        if self.kind == "shift":
            return "wkv_token_shift" + bf
        if self.gated:
            return f"wkv_forward{bf}_gated"
        return f"wkv_forward{bf}_state" if self.has_state else f"wkv_forward{bf}"

    def call(self, d, stream=None):
        """One C-ABI call on `stream` (default: torch's current stream, the
        capture stream while a graph is being captured) over the buffers `d`."""
        lib = self.lib
        sh = (stream or self.torch.cuda.current_stream()).cuda_stream
        B, T, C = self.B, self.T, self.C
        fn = getattr(lib, self.api())
        if self.kind == "scan":
            return fn(B, T, C, d["a"].data_ptr(), d["b"].data_ptr(), None, d["h"].data_ptr(), sh)
        if self.kind == "lru":
            k = self.consts
            return fn(B, T, C, k["nu_log"].data_ptr(), k["theta_log"].data_ptr(),
                      k["gamma"].data_ptr(), d["u"].data_ptr(), None, d["x"].data_ptr(), sh)
        if self.kind == "shift":   # last token handed on in place
            return fn(B, T, C, self.n_mix, d["x"].data_ptr(), d["xp"].data_ptr(),
                      self.consts["mu"].data_ptr(), d["out"].data_ptr(), d["xp"].data_ptr(), sh)
        w, u = self.consts["w"].data_ptr(), self.consts["u"].data_ptr()
        if self.kind == "bwd":
            return fn(B, T, C, w, u, d["k"].data_ptr(), d["v"].data_ptr(), d["gy"].data_ptr(),
                      d["gk"].data_ptr(), d["gv"].data_ptr(), d["gw"].data_ptr(),
                      d["gu"].data_ptr(), sh)
        s = d["s"].data_ptr() if self.has_state else None   # state updated in place
        if self.gated:
            return fn(B, T, C, w, u, d["k"].data_ptr(), d["v"].data_ptr(), d["r"].data_ptr(),
                      d["y"].data_ptr(), s, s, sh)
        if self.has_state:
            return fn(B, T, C, w, u, d["k"].data_ptr(), d["v"].data_ptr(), d["y"].data_ptr(),
                      s, s, sh)
        return fn(B, T, C, w, u, d["k"].data_ptr(), d["v"].data_ptr(), d["y"].data_ptr(), sh)

    def launches_per_step(self):
        """Kernels one step launches: the gradient path runs four when a
        tensor map describes its rows (forward states and reverse segment
        summaries, reverse carries, gradients, reduction), six otherwise;
        every other path one."""
        if self.kind == "bwd":
            return 4 if (self.C * 4) % 16 == 0 else 6
        return 1

    def kernel(self):
        """The dominant kernel a step launches (the library's dispatch rule)."""
        if self.kind == "shift":
            return "token_shift_kernel"
        if self.kind == "bwd":
            return ("wkv_bwd_* (%d kernels per step, timed together)" % self.launches_per_step())
        if self.kind == "wkv" and self.T <= 16:
            return "wkv_serial_kernel"
        lt = self.lib.wkv_tile_steps_for(self.B, self.T, self.C, min(self.es, 4))
        if lt in (8, 32):
            return "chunked_scan_kernel"
        if self.kind == "wkv" and self.dtype == "f32" and -(-self.T // lt) <= 16 and \
                not (self.gated and lt == 256):
            return "persistent_wkv_kernel"
        return "persistent_scan_kernel"

    def step(self, i):
        st = self.call(self.sets[i % self.n_sets])
        if st != 0:
            raise RuntimeError(f"library call failed: {st}: {self.lib.wkv_last_error().decode()}")


def time_steps(torch, wl, K):
    """K steps launched directly, back to back; events around the whole region
    and around every launch.  When the host is slower than the GPU these
    per-launch events also see host time, so `time_steps_graph` is the
    default."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    start.record(stream)
    for i in range(K):
        ev[i][0].record(stream)
        wl.step(i)
        ev[i][1].record(stream)
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end), [a.elapsed_time(b) for a, b in ev]


class StepGraphs:
    """Steps captured into CUDA graphs (each step one C-ABI call), so K steps
    replay back to back on the device with no host work between them.  Events
    on the launching stream bracket every replay; a launch's duration is its
    replay's duration over the steps in it."""

    def __init__(self, torch, wl, K, chunk=128):
        self.torch, self.wl, self.K = torch, wl, K
        self.G = min(K, chunk)
        self.reps, self.tail = divmod(K, self.G)
        self.side = torch.cuda.Stream()
        self.graph = self._capture(self.G)
        self.tail_graph = self._capture(self.tail) if self.tail else None

    def _capture(self, n):
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        # the library keeps one look-back workspace per stream and cannot
        # allocate it during capture: size it with plain calls first
        torch.cuda.synchronize()
        with torch.cuda.stream(self.side):
            for i in range(3):
                self.wl.step(i)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=self.side):
            for i in range(n):
                self.wl.step(i)
        torch.cuda.synchronize()
        return g

    def warm(self):
        self.graph.replay()
        if self.tail_graph is not None:
            self.tail_graph.replay()
        self.torch.cuda.synchronize()

    def run(self):
        """Replay K steps; total ms and the mean launch ms of every replay."""
        torch = self.torch
        stream = torch.cuda.current_stream()
        mk = lambda: torch.cuda.Event(enable_timing=True)   # noqa: E731
        marks = [mk() for _ in range(self.reps + 2)]
        marks[0].record(stream)
        for r in range(self.reps):
            self.graph.replay()
            marks[r + 1].record(stream)
        if self.tail_graph is not None:
            self.tail_graph.replay()
        marks[-1].record(stream)
        marks[-1].synchronize()
        per = [marks[r].elapsed_time(marks[r + 1]) / self.G for r in range(self.reps)]
        return marks[0].elapsed_time(marks[-1]), per


def host_overhead_us(torch, wl, n=200):
    """Host time of one C-ABI call (argument checks, tensor maps, launch),
    measured while the GPU is busy so calls never wait on the device."""
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(n):
        wl.step(i)
    dt = time.perf_counter() - t0
    torch.cuda.synchronize()
    return dt / n * 1e6


def e2e_leg(torch, wl, steps):
    """End to end through the library with host buffers, timed with CUDA
    events on the current stream around synchronous steps.  WKV and the scan
    go through the library's host-buffer entry points (upload, compute and
    download overlapped in chunks inside the call).  The entry points with no
    host-buffer form (state, gate, token shift) run as a user would: pinned
    host -> device copies of the step's inputs, the device call, device ->
    host copies of its outputs, on one stream, synchronised."""
    lib = wl.lib
    pinned = {k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory() for k, v in wl.host.items()}
    outs = {k: torch.empty(shape, dtype=torch.int16 if wl.dtype == "bf16" else torch.float32
                           ).pin_memory() for k, shape in wl.outputs.items()}
    hp = {k: t.cpu().pin_memory() for k, t in wl.consts.items()}
    host_api = (wl.kind == "scan" and wl.dtype == "f32") or \
        (wl.kind == "wkv" and not wl.gated and not wl.has_state)
    if host_api:
        if wl.kind == "scan":
            api = "diag_scan_host"
            call = lambda: lib.diag_scan_host(wl.B, wl.T, wl.C, pinned["a"].data_ptr(),  # noqa: E731
                                              pinned["b"].data_ptr(), None, outs["h"].data_ptr())
        else:
            api = "wkv_forward_bf16_host" if wl.dtype == "bf16" else "wkv_forward_host"
            fn = getattr(lib, api)
            call = lambda: fn(wl.B, wl.T, wl.C, hp["w"].data_ptr(), hp["u"].data_ptr(),  # noqa: E731
                              pinned["k"].data_ptr(), pinned["v"].data_ptr(),
                              outs["y"].data_ptr())
        h2d = sum(t.numel() * t.element_size() for t in pinned.values()) + \
            sum(t.numel() * t.element_size() for t in hp.values())
        d2h = sum(t.numel() * t.element_size() for t in outs.values())
    else:
        api = wl.api() + " with pinned copies on one stream"
        d = {k: torch.empty(t.shape, dtype=t.dtype, device=wl.dev) for k, t in pinned.items()}
        d.update({k: torch.empty(t.shape, dtype=t.dtype, device=wl.dev) for k, t in outs.items()})
        if wl.dtype == "bf16":   # bf16 storage travels as int16 bits
            d = {k: (t.view(torch.bfloat16) if t.dtype == torch.int16 else t)
                 for k, t in d.items()}
        back = dict(outs)
        # in-place state / last token comes back too
        for k in ("s", "xp"):
            if k in pinned:
                back[k] = pinned[k]

        def call():
            stream = torch.cuda.current_stream()
            for k, t in pinned.items():
                d[k].view(t.dtype).copy_(t, non_blocking=True)
            st = wl.call(d, stream)
            for k, t in back.items():
                t.copy_(d[k].view(t.dtype), non_blocking=True)
            stream.synchronize()
            return st
        h2d = sum(t.numel() * t.element_size() for t in pinned.values())
        d2h = sum(t.numel() * t.element_size() for t in back.values())

    def one():
        st = call()
        if st != 0:
            raise RuntimeError(f"{api} failed: {st}: {lib.wkv_last_error().decode()}")

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    t0 = time.perf_counter()
    a.record(stream)
    for _ in range(steps):
        one()
    b.record(stream)
    b.synchronize()
    wall_ms = (time.perf_counter() - t0) / steps * 1e3
    ms = a.elapsed_time(b) / steps
    return {"value": wl.elements / (ms / 1e3), "unit": "elem/s", "ms_per_step": ms,
            "wall_ms_per_step": wall_ms, "steps": steps, "api": api,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "host_buffers": "pinned"}


# ---------------------------------------------------------------------------
# CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------
def oracle_runner(name, max_elements=None, nthreads=0):
    """A callable running the float64 oracle once over a sample of the
    workload, and the sample's element count and description.  `nthreads`
    (0: all) is passed to the C oracle's OpenMP loops; the numpy oracles
    (gate, token shift, LRU) run on one thread either way."""
    import oracle
    spec = workloads.WORKLOADS[name]
    if isinstance(spec, workloads.ScanSpec):
        x = workloads.make_scan(name)
        a, b = x.a.astype(np.float64), x.b.astype(np.float64)
        B, T, C = a.shape
        rows = B if max_elements is None else max(1, min(B, max_elements // (T * C)))
        a, b = np.ascontiguousarray(a[:rows]), np.ascontiguousarray(b[:rows])
        fn = lambda: oracle.scan_rnn(a, b, None, nthreads)   # noqa: E731
        return fn, rows * T * C, f"{rows} of {B} batch rows (all T={T}, D={C})"
    if isinstance(spec, workloads.LruSpec):
        x = workloads.make_lru(name)
        B, T, C = x.u.shape[:3]
        rows = B if max_elements is None else max(1, min(B, max_elements // (T * C)))
        u = x.u_complex()[:rows]
        fn = lambda: oracle.lru_scan(x.nu_log, x.theta_log, x.gamma, u)   # noqa: E731
        return fn, rows * T * C, f"{rows} of {B} batch rows (all T={T}, D={C} complex)"
    if isinstance(spec, workloads.ShiftSpec):
        x = workloads.make_token_shift(name)
        B, T, C = x.x.shape
        rows = B if max_elements is None else max(1, min(B, max_elements // (T * C)))
        xs = np.ascontiguousarray(x.x[:rows], dtype=np.float64)
        xp = np.ascontiguousarray(x.x_prev[:rows], dtype=np.float64)
        mu = x.mu.astype(np.float64)
        fn = lambda: oracle.token_shift(xs, mu, xp)   # noqa: E731
        return fn, rows * T * C, f"{rows} of {B} batch rows (all T={T}, C={C})"
    x = workloads.make_wkv(name)
    k, v = x.k.astype(np.float64), x.v.astype(np.float64)
    w, u = x.w.astype(np.float64), x.u.astype(np.float64)
    B, T, C = k.shape
    rows, chans = B, C
    if max_elements is not None:
        rows = max(1, min(B, max_elements // (T * C)))
        if rows * T * C > max_elements:   # even one row is too much: fewer channels
            chans = max(1, min(C, max_elements // T))
    k = np.ascontiguousarray(k[:rows, :, :chans]); v = np.ascontiguousarray(v[:rows, :, :chans])
    w, u = w[:chans], u[:chans]
    s_in = None if x.s_in is None else \
        np.ascontiguousarray(x.s_in[:rows, :, :chans], dtype=np.float64)
    if x.gy is not None:
        gy = np.ascontiguousarray(x.gy[:rows, :, :chans], dtype=np.float64)
        fn = lambda: oracle.wkv_backward_rnn(w, u, k, v, gy, nthreads)   # noqa: E731
    elif x.r is not None:
        r = np.ascontiguousarray(x.r[:rows, :, :chans], dtype=np.float64)
        fn = lambda: oracle.wkv_gated(w, u, k, v, r, s_in)   # noqa: E731
    elif s_in is not None:
        fn = lambda: oracle.wkv_rnn_state(w, u, k, v, s_in, nthreads)   # noqa: E731
    else:
        fn = lambda: oracle.wkv_rnn(w, u, k, v, nthreads)   # noqa: E731
    return fn, rows * T * chans, f"{rows} of {B} batch rows x {chans} of {C} channels (all T={T})"


def _time_oracle(name, seconds, nthreads):
    """Run the oracle over a sample of `name` for about `seconds`; elements
    per second, the thread count used and the sample's description."""
    import oracle
    fn, n, desc = oracle_runner(name, max_elements=None, nthreads=nthreads)
    t0 = time.perf_counter(); fn(); one = time.perf_counter() - t0
    if one > seconds:   # a smaller sample of the same workload
        fn, n, desc = oracle_runner(name, max_elements=max(1, int(n * seconds / one / 2)),
                                    nthreads=nthreads)
        t0 = time.perf_counter(); fn(); one = time.perf_counter() - t0
    reps = max(1, int(seconds / max(one, 1e-6)))
    t0 = time.perf_counter()
    for _ in range(reps):
        fn()
    dt = time.perf_counter() - t0
    spec = workloads.WORKLOADS[name]
    numpy_only = isinstance(spec, (workloads.LruSpec, workloads.ShiftSpec)) or \
        (isinstance(spec, workloads.WkvSpec) and spec.gated)
    cores = 1 if (nthreads == 1 or numpy_only) else oracle.max_threads()
    return {"value": n * reps / dt, "cores": cores,
            "sample": f"{desc}, {reps} passes, float64 RNN-mode oracle", "seconds": dt}


def cpu_baseline(name, seconds):
    """The float64 oracle on all of this host's cores, and on one core."""
    allc = _time_oracle(name, seconds, 0)
    one = _time_oracle(name, seconds, 1)
    return {"value": allc["value"], "unit": "elem/s", "cores": allc["cores"],
            "kind": "oracle", "sample": allc["sample"], "seconds": allc["seconds"],
            "cpu": cpu_model(),
            "one_core": {"value": one["value"], "unit": "elem/s", "cores": 1,
                         "sample": one["sample"], "seconds": one["seconds"]}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    budget = 150.0   # whole run within a few minutes
    fn, n, desc = oracle_runner(args.workload)
    t0 = time.perf_counter(); fn(); one = time.perf_counter() - t0
    per_step = budget / max(1, args.steps + args.warmup)
    if one > per_step:
        fn, n, desc = oracle_runner(args.workload, max_elements=max(1, int(n * per_step / one)))
    for _ in range(args.warmup):
        fn()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn()
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    spec = workloads.WORKLOADS[args.workload]
    line = {
        "impl": "reference", "metric": metric_for(spec), "value": value, "unit": "elem/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(spec, args.workload),
        "cpu_baseline": {"value": value, "unit": "elem/s", "cores": oracle.max_threads(),
                         "kind": "oracle", "sample": f"{desc} per step, float64 oracle"},
        "e2e": {"value": value, "unit": "elem/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(dist, value, device):
    """The largest `value` over all ranks (every rank gets it)."""
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(elements_per_rank, world, ms_per_step):
    """Whole-job throughput: every rank processes its own copy of the
    workload each step (weak scaling); the step time is the slowest rank's."""
    return elements_per_rank * world / (ms_per_step / 1e3)


def workload_config(spec, name):
    if isinstance(spec, workloads.LruSpec):
        return {"workload": name, "op": "lru_scan (complex diagonal recurrence)", "B": spec.B,
                "T": spec.T, "D": spec.D, "io": "complex64"}
    if isinstance(spec, workloads.ScanSpec):
        return {"workload": name, "op": "diag_scan" + ("_bf16" if spec.dtype == "bf16" else "") +
                f" ({spec.form} form)", "B": spec.B, "T": spec.T, "D": spec.D, "io": spec.dtype}
    bf = "_bf16" if spec.dtype == "bf16" else ""
    if isinstance(spec, workloads.ShiftSpec):
        return {"workload": name, "op": f"wkv_token_shift{bf} ({spec.n_mix} mixing vectors, "
                "last token read and written in place)", "B": spec.B, "T": spec.T, "C": spec.C,
                "io": spec.dtype}
    if spec.backward:
        op = "wkv_backward (gk, gv, gw, gu for an upstream gradient)"
    elif spec.gated:
        op = f"wkv_forward{bf}_gated (sigma(r) * wkv in one pass)"
    elif spec.state:
        op = f"wkv_forward{bf}_state (state [B,3,C] fp32 read and written in place)"
    else:
        op = f"wkv_forward{bf}"
    return {"workload": name, "op": op, "B": spec.B, "T": spec.T, "C": spec.C, "io": spec.dtype}


def metric_for(spec):
    if isinstance(spec, workloads.WkvSpec) and spec.backward:
        return "WKV backward B·T·C elems/s and achieved HBM GB/s vs B200 peak (1 GPU)"
    if isinstance(spec, workloads.LruSpec):
        return "LRU scan B·T·D complex elems/s and achieved HBM GB/s vs B200 peak (1 GPU)"
    if isinstance(spec, workloads.ShiftSpec):
        return "token shift B·T·C elems/s and achieved HBM GB/s vs B200 peak (1 GPU)"
    return METRIC


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------
def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist

    import rwkv_wkv_mixing_b200 as wkv
    props = torch.cuda.get_device_properties(local)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    if args.tile_steps:
        wkv.wkv_set_tile_steps(args.tile_steps)
    shape = tuple(int(v) for v in args.shape.split(",")) if args.shape else None
    if shape is not None and len(shape) != 3:
        raise SystemExit("--shape takes three integers: B,T,C")
    wl = DeviceWorkload(args.workload, torch, wkv.lib, l2, shape)

    def barrier():
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    # warm-up, then an untimed soak so clocks and caches reach steady state
    for i in range(args.warmup):
        wl.step(i)
    torch.cuda.synchronize()
    wkv.wkv_device_status()
    uuid = None
    try:
        uuid = "GPU-" + str(props.uuid)
    except Exception:
        pass
    sampler = None if args.no_clocks else ClockSampler(uuid)
    t_soak = time.time()
    if args.soak_seconds > 0:
        t_end = time.time() + args.soak_seconds
        i = 0
        while time.time() < t_end:
            for _ in range(64):
                wl.step(i); i += 1
            torch.cuda.synchronize()

    graphs = None
    if args.launch == "graph":
        graphs = StepGraphs(torch, wl, args.steps)
        graphs.warm()
    host_us = host_overhead_us(torch, wl)

    barrier()
    if sampler is not None:
        sampler.fast(True)
    t_timed0 = time.time()
    if graphs is not None:
        total_ms, per = graphs.run()
    else:
        total_ms, per = time_steps(torch, wl, args.steps)
    t_timed1 = time.time()
    barrier()
    if sampler is not None:
        sampler.fast(False)
        sampler.stop()
    wkv.wkv_device_status()   # raises if a device-side wait gave up

    if pg is not None:
        total_ms = max_over_ranks(pg, total_ms, "cuda")

    ms_per_step = total_ms / args.steps
    value = aggregate_rate(wl.elements, world, ms_per_step)
    if not per:
        per = [total_ms / args.steps]
    launch_ms = statistics.mean(per)
    peak, peak_kind = read_peaks()
    achieved = wl.alg_bytes / (launch_ms / 1e3) / 1e9
    traffic = recorded_traffic(args.workload)

    e2e = None
    if not args.no_e2e:
        e2e = e2e_leg(torch, wl, args.e2e_steps)
        if pg is not None:
            e2e["ms_per_step"] = max_over_ranks(pg, e2e["ms_per_step"], "cuda")
            e2e["value"] = aggregate_rate(wl.elements, world, e2e["ms_per_step"])
        wkv.wkv_device_status()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(args.workload, args.cpu_seconds)

    spec = wl.spec
    cfg = workload_config(spec, args.workload)
    if shape is not None:
        cfg.update({"B": wl.B, "T": wl.T, ("D" if "D" in cfg else "C"): wl.C,
                    "shape": "overridden by --shape (not the named workload's size)"})
    cfg.update({"parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                "l2": (f"inputs rotate over {wl.n_sets} buffer sets "
                       f"({wl.n_sets * wl.set_bytes / 1e6:.0f} MB > L2 "
                       f"{l2 / 1e6:.0f} MB)"),
                "tile_steps": wkv.wkv_tile_steps_for(wl.B, wl.T, wl.C, min(wl.es, 4)),
                "launch": args.launch + (" (K steps replayed from captured graphs)"
                                         if args.launch == "graph" else ""),
                "gpu": props.name, "sms": props.multi_processor_count})
    line = {
        "metric": metric_for(wl.spec), "value": value, "unit": "elem/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic (seeded, distributions of the named workload)",
        "config": cfg,
        "hbm_gbs": wl.alg_bytes * world / (ms_per_step / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_kind,
                     "traffic": traffic, "alg_bytes_per_launch": wl.alg_bytes,
                     "launch_ms_mean": launch_ms,
                     "launch_ms_median": statistics.median(per),
                     "kernel": wl.kernel()},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * wl.launches_per_step(),
        "host_us_per_call": host_us,
        "clocks": (sampler.summary(t_timed0, t_timed1, total_ms) if sampler is not None
                   else None),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
