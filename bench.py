"""Benchmark of the Hadamard-rotated W4A4 quantized linear layer on B200.

One step = one pass of the hot path over one batch: the fused rotate-quantize
kernel on the bf16 activations (qs_quant_act) followed by the tcgen05 integer
GEMM with the dequantizing epilogue (qs_qlinear).  The weights are packed once
beforehand (qs_pack_weights is offline preparation, not part of a step).

Workload: the Wan2.1-14B-like FFN up-projection, M = 32760 tokens,
K = 5120, N = 13824, W4A4, clip ratio 0.9, seed 2 (synthetic inputs, see
bit_quantized_linear_hadamard_b200/inputs.py).  The activations (335 MB bf16)
and the output (906 MB bf16) are larger than the 126 MB L2, so no L2 flush
is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 it is launched by torchrun, one process per GPU; every rank runs the
same single-GPU workload (replicas: the layer shards by tokens with no
collective), the time is the max over ranks, and `value` counts the work of
all ranks.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4 qlinear TOPS and tokens/s at Wan-14B FFN shape; % of INT8 peak / HBM"
UNIT = "TOPS"
PROFILES = os.path.join(ROOT, "profiles")
# The dense int8 tensor peak is taken as the measured dense bf16 GEMM peak times
# the nominal int8:bf16 dense ratio of B200 (4.5 / 2.25 = 2).
INT8_PER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--e2e-chunks", type=int, default=16,
                   help="token chunks of the end-to-end step: the host->device copy, the layer "
                        "and the device->host copy of consecutive chunks overlap on 3 streams")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extras", action="store_true",
                   help="skip the per-config table and the quality report")
    p.add_argument("--tokens", type=int, default=None,
                   help="override M (profiling captures of a smaller case of the same shape)")
    p.add_argument("--workload", default=None,
                   help="the Wan FFN variant to time: w4a4 (default), w8a8, w4a8 or w4a6")
    p.add_argument("--act-codes", choices=["bytes", "packed"], default="packed",
                   help="storage of 4-bit activation codes: two per byte (packed int4, "
                        "widened in the GEMM's shared memory) or one per byte (loaded by TMA "
                        "straight into the operand tiles)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# the sources of each headline kernel and its launch (the kernel's file and
# the shared helpers): counters taken on other sources are not reported
KERNEL_SOURCES = {
    "qgemm_kernel": ("qs_gemm.cuh", "qs_host.cuh", "qs_ptx.cuh"),
    "rotate_quant_kernel": ("qs_host.cuh", "qs_ptx.cuh", "qs_quant.cuh"),
}
HEADLINE_SOURCES = ("qs_gemm.cuh", "qs_host.cuh", "qs_ptx.cuh", "qs_quant.cuh")


def gemm_kernel(sx: int, sw: int) -> tuple[str, str]:
    """(kernel family as keyed in the ncu record, instantiation) of the GEMM
    that the storage widths sx (activations) and sw (weights) run."""
    return "qgemm_kernel", f"qgemm_kernel<{sx},{sw},false,false> (tcgen05 kind::i8)"


def source_hash(names, read=None) -> str:
    """sha256 over (name, contents) of the given csrc files, 16 hex digits;
    `read(name) -> bytes` supplies the contents (default: the files here)."""
    csrc = os.path.join(ROOT, "bit_quantized_linear_hadamard_b200", "csrc")
    if read is None:
        def read(name):
            with open(os.path.join(csrc, name), "rb") as f:
                return f.read()
    h = hashlib.sha256()
    for name in names:
        h.update(name.encode() + read(name))
    return h.hexdigest()[:16]


def kernel_source_hash(kernel: str | None = None) -> str:
    """Hash of one headline kernel's sources, or of all of them."""
    return source_hash(HEADLINE_SOURCES if kernel is None else KERNEL_SOURCES[kernel])


def ncu_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` in `workload` from the committed ncu
    summary, or None if there is none or the kernel's sources changed since
    the counters were taken."""
    path = os.path.join(PROFILES, "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    hashes = d.get("source_hashes")
    if hashes is not None:
        if kernel not in KERNEL_SOURCES or hashes.get(kernel) != kernel_source_hash(kernel):
            return None
    elif d.get("source_hash") != kernel_source_hash():
        return None
    k = d.get("workloads", {}).get(workload, {}).get(kernel)
    return None if k is None else k.get("dram_bytes_per_launch_full")


def workload_line_config(cfg, act_codes: str, world: int, M: int | None = None) -> dict:
    """The `config` object of a bench line: the same keys and values for this
    library's arm and the oracle arm of one workload."""
    return {"workload": cfg.name, "M": cfg.M if M is None else M, "K": cfg.K, "N": cfg.N,
            "bits_w": cfg.bits, "bits_x": cfg.act_bits, "alpha": cfg.alpha,
            "act_codes": act_codes if cfg.act_bits == 4 else "bytes",
            "seed": cfg.seed, "parallelism": f"replicas{world}",
            "l2": "inputs larger than L2 (x 335 MB, out 906 MB bf16); no flush"}


def workload_config(I, name):
    """The Wan-14B FFN up-projection config the step runs (W4A4 by default)."""
    table = {"w4a4": I.WAN_FFN, "w8a8": I.WAN_FFN_W8, "w4a8": I.WAN_FFN_W4A8,
             "w4a6": I.WAN_FFN_W4A6}
    if name is None:
        return I.WAN_FFN
    for key, cfg in table.items():
        if name in (key, cfg.name):
            return cfg
    raise SystemExit(f"unknown workload {name!r}; choose one of {sorted(table)}")


class ClockSampler:
    """SM clock, power and clock-event reasons of the GPU under test, read on a
    host thread every millisecond through NVML (reads only; nvidia-smi if NVML
    is not available).  Only the samples taken between mark_start() and
    mark_end(), i.e. during the timed region, are reported."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.nv = None
        self.samples = []
        self.t_on = self.t_off = None

    def _handle(self, nv):
        """The NVML handle of CUDA device `index` (by UUID: CUDA and NVML may
        number the devices differently)."""
        try:
            import torch
            u = str(getattr(torch.cuda.get_device_properties(self.index), "uuid", ""))
        except Exception:  # noqa: BLE001 - no CUDA device: NVML's numbering
            u = ""
        for cand in ((u, "GPU-" + u) if u else ()):
            try:
                return nv.nvmlDeviceGetHandleByUUID(cand)
            except Exception:  # noqa: BLE001 - try the next form
                pass
        return nv.nvmlDeviceGetHandleByIndex(self.index)

    def start(self):
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            self.h = self._handle(nv)
            self.nv = nv
            reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.stop_flag = False

            def loop():
                while not self.stop_flag:
                    try:
                        self.samples.append((time.perf_counter(),
                                             nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                             reasons(self.h),
                                             nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0))
                    except Exception:  # noqa: BLE001 - a failed read is skipped
                        pass
                    time.sleep(0.001)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:  # noqa: BLE001 - no NVML: nvidia-smi
            self.nv = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def mark_start(self):
        self.t_on = time.perf_counter()

    def mark_end(self):
        self.t_off = time.perf_counter()

    def stop(self):
        if self.nv is not None:
            time.sleep(0.01)
            self.stop_flag = True
            self.thread.join(timeout=2)
            nv = self.nv
            mx = float(nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM))
            inside = [r for r in self.samples
                      if self.t_on is not None and self.t_on <= r[0] <= (self.t_off or r[0])]
            rows = inside or self.samples
            if not rows:
                return None
            reasons = sorted({name for r in rows for bit, name in self.REASONS.items()
                              if r[2] & bit})
            return {"sm_mhz": statistics.median(float(r[1]) for r in rows), "sm_max_mhz": mx,
                    "reasons": reasons, "samples": len(rows),
                    "power_w_max": max(r[3] for r in rows),
                    "source": "nvml, 1 ms, " + ("timed region" if inside else "whole run")}
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [l.split(", ") for l in out.strip().splitlines() if l.strip()]
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        if not sm:
            return None
        mx = max(float(r[2]) for r in rows if len(r) >= 9 and r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows if len(r) >= 9 for i in range(4)
                          if r[5 + i].strip() == "Active"})
        loaded = [v for v in sm if v > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(sm), "power_w_max": max(float(r[3]) for r in rows
                                                       if len(r) >= 9 and _isnum(r[3])),
                "source": "nvidia-smi, 100 ms, whole run"}


def _isnum(s):
    try:
        float(s)
        return True
    except ValueError:
        return False


class OracleSample:
    """The oracle as it stands, on the host cores, on a bounded sample of the
    workload: `rows` tokens through quant_act + int GEMM + epilogue against
    the full weight (weight packing is offline, done once and not timed)."""

    def __init__(self, d, bits, alpha, bits_x=None):
        from bit_quantized_linear_hadamard_b200 import inputs as I
        from oracle import qs_oracle as O
        self.O, self.bits, self.alpha = O, bits, alpha
        self.bits_x = bits if bits_x is None else bits_x
        self.x = d["x"]
        self.qw, self.sw = O.pack_weights(I.bf16_bits(d["w"]), bits)
        self.bb = I.bf16_bits(d["bias"])
        self.bf16_bits = I.bf16_bits
        self.K, self.N = d["x"].shape[1], d["w"].shape[0]

    def run(self, rows: int) -> float:
        xb = self.bf16_bits(self.x[:rows])
        t0 = time.perf_counter()
        qa, sa = self.O.quant_act(xb, self.bits_x, self.alpha)
        acc = self.O.int_gemm(qa, self.qw)
        self.O.epilogue(acc, sa, self.sw, self.bb)
        return time.perf_counter() - t0

    def baseline(self, rows: int = 128, rows_per_core: int = 64) -> dict:
        """All host cores (one oracle process per core on its own token
        block) as the value, the one-thread run beside it."""
        dt = self.run(rows)
        ops = 2.0 * rows * self.N * self.K
        single = {"value": ops / dt / 1e12, "unit": UNIT, "cores": 1,
                  "sample": f"first {rows} tokens, one host thread, {dt:.2f} s",
                  "tokens_per_s": rows / dt}
        pool = OraclePool(self)
        try:
            prow, pdt = pool.run(rows_per_core)
        finally:
            pool.close()
        pops = 2.0 * prow * self.N * self.K
        return {"value": pops / pdt / 1e12, "unit": UNIT, "cores": pool.procs, "kind": "oracle",
                "host": host_info(),
                "sample": f"{prow} of {self.x.shape[0]} tokens ({rows_per_core} per process, "
                          f"{pool.procs} processes, one per host core, each numpy on one "
                          f"thread), full K={self.K}, N={self.N} (quant_act + int GEMM + "
                          f"epilogue), {pdt:.2f} s wall",
                "tokens_per_s": prow / pdt, "single_core": single}


def _oracle_worker_init(qw, sw, bb, bits_x, alpha):
    global _OW
    from oracle import qs_oracle as O
    _OW = (O, qw, sw, bb, bits_x, alpha)


def _oracle_worker(xb):
    O, qw, sw, bb, bits_x, alpha = _OW
    t0 = time.perf_counter()
    qa, sa = O.quant_act(xb, bits_x, alpha)
    acc = O.int_gemm(qa, qw)
    O.epilogue(acc, sa, sw, bb)
    return time.perf_counter() - t0


class OraclePool:
    """One spawned oracle process per host core (spawned, not forked: the
    parent has a CUDA context), each with one BLAS/OpenMP thread."""

    def __init__(self, sample: "OracleSample", procs: int | None = None):
        import multiprocessing as mp
        self.sample = sample
        self.procs = procs or os.cpu_count() or 1
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS",
                                                  "MKL_NUM_THREADS")}
        for k in saved:
            os.environ[k] = "1"
        try:
            self.pool = mp.get_context("spawn").Pool(
                self.procs, initializer=_oracle_worker_init,
                initargs=(sample.qw, sample.sw, sample.bb, sample.bits_x, sample.alpha))
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        # every worker imports numpy and the oracle before anything is timed
        self.pool.map(_oracle_worker, [sample.bf16_bits(sample.x[:2])] * self.procs)

    def run(self, rows_per_proc: int) -> tuple[int, float]:
        """Token blocks of `rows_per_proc` rows, one per process, all at once:
        returns (rows, wall seconds)."""
        blocks = []
        M = self.sample.x.shape[0]
        for i in range(self.procs):
            r0 = (i * rows_per_proc) % max(1, M - rows_per_proc)
            blocks.append(self.sample.bf16_bits(self.sample.x[r0:r0 + rows_per_proc]).copy())
        t0 = time.perf_counter()
        self.pool.map(_oracle_worker, blocks, chunksize=1)
        return rows_per_proc * self.procs, time.perf_counter() - t0

    def close(self):
        self.pool.close()
        self.pool.join()


def host_info() -> dict:
    """The host the oracle ran on: its core count and CPU model."""
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def combine_ranks(times_ms, steps, ops_per_step, world, device="cpu"):
    """Replicas: every rank ran the same single-GPU workload.  The job's time is
    the max over ranks of each timing; the value counts all ranks' work."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(list(times_ms), dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    times = t.tolist()
    ms_per_step = times[0] / steps
    return {"times_ms": times, "ms_per_step": ms_per_step,
            "value": ops_per_step * world / (ms_per_step * 1e-3) / 1e12}


def time_layer(qs, torch, x, wp, ws, bias, bits, alpha, stream, steps=5, warmup=2, bits_x=None,
               x_flags=0):
    """Mean CUDA-event times (ms) of the activation kernel and the GEMM for one
    layer; ``bits`` is the weights' code width, ``bits_x`` the activations',
    ``x_flags`` their quantisation flags (storage)."""
    bx = bits if bits_x is None else bits_x
    sx = qs.storage_bits(bx, x_flags)
    M, K = x.shape
    N = wp.shape[0]
    dev = x.device
    xp = torch.empty((M, qs.packed_cols(K, bx, x_flags)), dtype=torch.uint8, device=dev)
    xs = torch.empty((M,), dtype=torch.float32, device=dev)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    for _ in range(warmup):
        qs.qs_quant_act(x, M, K, bx, alpha, x_flags, xp, xs, stream)
        qs.qs_qlinear_mixed(xp, xs, sx, wp, ws, bits, bias, M, N, K, out, stream)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for e in ev:
        e[0].record(stream)
        qs.qs_quant_act(x, M, K, bx, alpha, x_flags, xp, xs, stream)
        e[1].record(stream)
        qs.qs_qlinear_mixed(xp, xs, sx, wp, ws, bits, bias, M, N, K, out, stream)
        e[2].record(stream)
    stream.synchronize()
    q = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
    g = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
    return q, g, out


def time_quant_alone(qs, torch, x, bx, alpha, x_flags, stream, launches=20, warmup=3):
    """Mean CUDA-event time (ms) of the activation kernel launched back to back
    on its own (no GEMM between launches: none of the GEMM's output lines are
    still being written back from L2 while it streams x)."""
    M, K = x.shape
    xp = torch.empty((M, qs.packed_cols(K, bx, x_flags)), dtype=torch.uint8, device=x.device)
    xs = torch.empty((M,), dtype=torch.float32, device=x.device)
    for _ in range(warmup):
        qs.qs_quant_act(x, M, K, bx, alpha, x_flags, xp, xs, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(launches):
        qs.qs_quant_act(x, M, K, bx, alpha, x_flags, xp, xs, stream)
    e1.record(stream)
    stream.synchronize()
    return e0.elapsed_time(e1) / launches


def all_configs(qs, torch, I, dev, stream):
    """Per-configuration throughput on one GPU (every seeded synthetic shape)."""
    res = {}
    runs = [(cfg, 0) for cfg in (*I.LAYER_CONFIGS, *I.MIXED_CONFIGS)]
    runs += [(cfg, qs.QS_FLAG_BYTE_CODES) for cfg in (I.HY_QKV, I.WAN_FFN)]
    for cfg, flags in runs:
        d = I.make_layer(cfg)
        with torch.cuda.stream(stream):
            x, w, b = d["x"].to(dev), d["w"].to(dev), d["bias"].to(dev)
            wp, ws = qs.pack_weights(w, cfg.bits, stream=stream)
        q, g, _ = time_layer(qs, torch, x, wp, ws, b, cfg.bits, cfg.alpha, stream,
                             bits_x=cfg.act_bits, x_flags=flags)
        name = cfg.name + ("_act_codes_in_bytes" if flags else "")
        res[name] = {"bits_w": cfg.bits, "bits_x": cfg.act_bits, "quant_ms": q, "gemm_ms": g,
                         "TOPS": cfg.ops / ((q + g) * 1e-3) / 1e12,
                         "gemm_TOPS": cfg.ops / (g * 1e-3) / 1e12,
                         "tokens_per_s": cfg.M / ((q + g) * 1e-3)}
        del x, w, b, wp, ws
    ch = I.make_chain(I.WAN_CHAIN)
    M = I.WAN_CHAIN.M
    layers, total, gelu_ms, ops, up_out = {}, 0.0, 0.0, 0, None
    for L in ch["layers"]:
        with torch.cuda.stream(stream):
            w, b = L["w"].to(dev), L["bias"].to(dev)
            wp, ws = qs.pack_weights(w, L["bits"], stream=stream)
            if L["x"] is not None:
                x = L["x"].to(dev)
            else:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                x = torch.empty_like(up_out)
                qs.gelu(up_out, stream=stream, out=x)
                e0.record(stream)
                for _ in range(5):
                    qs.gelu(up_out, stream=stream, out=x)
                e1.record(stream)
                stream.synchronize()
                gelu_ms = e0.elapsed_time(e1) / 5
        q, g, out = time_layer(qs, torch, x, wp, ws, b, L["bits"], ch["alpha"], stream)
        if L["name"] == "ffn_up":
            up_out = out
        lops = 2 * M * L["K"] * L["N"]
        ops += lops
        total += q + g
        layers[L["name"]] = {"bits": L["bits"], "K": L["K"], "N": L["N"], "quant_ms": q,
                             "gemm_ms": g, "TOPS": lops / ((q + g) * 1e-3) / 1e12}
    res[I.WAN_CHAIN.name] = {"bits_mask": ch["bits"], "layers": layers,
                             "tokens_per_s": M / (total * 1e-3),
                             "tokens_per_s_with_gelu": M / ((total + gelu_ms) * 1e-3),
                             "gelu_ms": gelu_ms, "TOPS": ops / (total * 1e-3) / 1e12}
    return res


def gbs_sequence(qs, torch, I, dev, stream, steps=8, delta=0.3):
    """δ-guided bit switching over consecutive steps of the Wan FFN layer:
    each step is the gated one-call layer plus the on-device distance update.
    The inputs drift by a seeded amount per step (synthetic stand-in for the
    denoising trajectory).  Returns per-step widths and times and the update
    kernel's time against HBM."""
    cfg = I.WAN_FFN
    d = I.make_layer(cfg)
    with torch.cuda.stream(stream):
        x = d["x"].to(dev)
        layer = qs.GbsLinear(d["w"].to(dev), d["bias"].to(dev), delta, cfg.alpha, stream=stream)
        g = torch.Generator(device=dev).manual_seed(cfg.seed)
        sigmas = [0.0, 0.01, 0.01, 0.3, 0.01, 0.02, 0.02, 0.2, 0.01, 0.01][:steps]
        widths, step_ms, upd_ms = [], [], []
        for t in range(steps):
            if t:
                x = (x.float() + sigmas[t] * torch.randn(x.shape, generator=g, device=dev,
                                                         dtype=torch.float32)).to(torch.bfloat16)
            stream.synchronize()
            widths.append(qs.gbs_state_host(layer.state)["bits"])
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            M = x.shape[0]
            if layer.workspace is None:
                layer.workspace = torch.empty((qs.qs_linear_workspace_bytes(M, cfg.K, 8),),
                                              dtype=torch.uint8, device=dev)
            out = torch.empty((M, cfg.N), dtype=torch.bfloat16, device=dev)
            e[0].record(stream)
            qs.qs_linear_gbs(x, M, cfg.K, cfg.alpha, layer.w4, layer.s4, layer.w8, layer.s8,
                             layer.bias, cfg.N, layer.state, layer.workspace,
                             layer.workspace.numel(), out, stream)
            e[1].record(stream)
            qs.qs_gbs_update(out, layer.prev, out.numel(), delta, layer.state, stream)
            e[2].record(stream)
            layer.prev = out
            stream.synchronize()
            step_ms.append(e[0].elapsed_time(e[2]))
            if t:
                upd_ms.append(e[1].elapsed_time(e[2]))
    n = cfg.M * cfg.N
    upd = sum(upd_ms) / len(upd_ms)
    pk, _ = peaks()
    return {"workload": cfg.name, "delta": delta, "sigmas": sigmas, "widths": widths,
            "step_ms": step_ms, "update_ms": upd,
            "update_GBps": 4.0 * n / (upd * 1e-3) / 1e9,
            "update_frac_hbm": 4.0 * n / (upd * 1e-3) / 1e9 / pk["hbm_gbs"],
            "update_bytes": 4 * n}


def bgr_layer(qs, torch, I, dev, stream, steps=5, warmup=2, rows=256):
    """The Wan FFN layer with weights on BGR grids (asymmetric, per channel):
    offline pack time, per-step times of the activation kernel (with code sums)
    and the asymmetric GEMM, and the output error against the symmetric weights
    on the first `rows` tokens."""
    cfg = I.WAN_FFN
    d = I.make_layer(cfg)
    M, K, N, bits, alpha = cfg.M, cfg.K, cfg.N, cfg.bits, cfg.alpha
    with torch.cuda.stream(stream):
        x, w, b = d["x"].to(dev), d["w"].to(dev), d["bias"].to(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        wp, ws, wo = qs.pack_weights_bgr(w, bits, 64, 8, stream=stream)
        e1.record(stream)
        stream.synchronize()
        pack_ms = e0.elapsed_time(e1)
        xp = torch.empty((M, qs.packed_cols(K, bits)), dtype=torch.uint8, device=dev)
        xs = torch.empty((M,), dtype=torch.float32, device=dev)
        xr = torch.empty((M,), dtype=torch.int32, device=dev)
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        for _ in range(warmup):
            qs.qs_quant_act_rowsum(x, M, K, bits, alpha, 0, xp, xs, xr, stream)
            qs.qs_qlinear_asym(xp, xs, xr, wp, ws, wo, b, M, N, K, bits, out, stream)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for e in ev:
            e[0].record(stream)
            qs.qs_quant_act_rowsum(x, M, K, bits, alpha, 0, xp, xs, xr, stream)
            e[1].record(stream)
            qs.qs_qlinear_asym(xp, xs, xr, wp, ws, wo, b, M, N, K, bits, out, stream)
            e[2].record(stream)
        stream.synchronize()
        q = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
        g = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
        ref = x[:rows].double() @ w.double().t() + b.double()
        wsp, wss = qs.pack_weights(w, bits, stream=stream)
        ysym = qs.qlinear(xp[:rows], xs[:rows], wsp, wss, b, bits, K, stream=stream).double()
        stream.synchronize()
    err = lambda y: float((y - ref).norm() / ref.norm())  # noqa: E731
    return {"workload": cfg.name + "_bgr", "candidates": 64, "iterations": 8,
            "pack_ms": pack_ms, "quant_rowsum_ms": q, "gemm_asym_ms": g,
            "TOPS": cfg.ops / ((q + g) * 1e-3) / 1e12, "gemm_TOPS": cfg.ops / (g * 1e-3) / 1e12,
            "rel_err_bgr": err(out[:rows].double()), "rel_err_symmetric": err(ysym),
            "error_rows": rows}


def sd4_layer(qs, torch, I, dev, stream, steps=5, warmup=2, rows=256):
    """The Wan FFN layer in SD4 (per-32-element mixed 4-bit formats): the
    weights quantised once, per step the activation quantiser and the
    decode-bf16 tensor-core GEMM; the output error on the first `rows` tokens
    against the unquantised layer, beside the W4A4 rotated layer's.  Also the
    activation decomposition of a seeded 1/16 of the tokens (their residual
    quantiser and the 2K-long GEMM over them) and its error on those tokens."""
    cfg = I.WAN_FFN
    d = I.make_layer(cfg)
    M, K, N = cfg.M, cfg.K, cfg.N
    with torch.cuda.stream(stream):
        x, w, b = d["x"].to(dev), d["w"].to(dev), d["bias"].to(dev)
        cw, mw = qs.sd4_quant(w, stream=stream)
        cx = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        mx = torch.empty((M, K // 32), dtype=torch.int16, device=dev)
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        for _ in range(warmup):
            qs.qs_sd4_quant(x, M, K, cx, mx, stream)
            qs.qs_sd4_linear(cx, mx, cw, mw, b, M, N, K, out, stream)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for e in ev:
            e[0].record(stream)
            qs.qs_sd4_quant(x, M, K, cx, mx, stream)
            e[1].record(stream)
            qs.qs_sd4_linear(cx, mx, cw, mw, b, M, N, K, out, stream)
            e[2].record(stream)
        stream.synchronize()
        q = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
        g = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
        # the weights decoded once (offline): only the activations decoded per
        # call; as bf16 (bf16 tensor cores) and as e4m3 bytes (block-scaled fp8)
        wdec = qs.sd4_decode(cw, mw, stream=stream)
        w8 = qs.sd4_decode_e4m3(cw, mw, stream=stream)
        out2 = torch.empty_like(out)
        out8 = torch.empty_like(out)
        qs.qs_sd4_linear_wdec(cx, mx, wdec, b, M, N, K, out2, stream)
        qs.qs_sd4_linear_e4m3w(cx, mx, w8, mw, b, M, N, K, out8, stream)

        def timed(fn):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            e[0].record(stream)
            for _ in range(steps):
                fn()
            e[1].record(stream)
            stream.synchronize()
            return e[0].elapsed_time(e[1]) / steps

        g2 = timed(lambda: qs.qs_sd4_linear_wdec(cx, mx, wdec, b, M, N, K, out2, stream))
        g8 = timed(lambda: qs.qs_sd4_linear_e4m3w(cx, mx, w8, mw, b, M, N, K, out8, stream))
        same = bool(torch.equal(out.view(torch.int16), out8.view(torch.int16)))
        # activations quantised straight to e4m3 bytes: nothing decoded in the GEMM
        x8 = torch.empty((M, K), dtype=torch.uint8, device=dev)
        m8 = torch.empty((M, K // 32), dtype=torch.int16, device=dev)
        out88 = torch.empty_like(out)
        qs.qs_sd4_quant_e4m3(x, M, K, x8, m8, stream)
        qs.qs_sd4_linear_e4m3(x8, m8, w8, mw, b, M, N, K, out88, stream)
        q8 = timed(lambda: qs.qs_sd4_quant_e4m3(x, M, K, x8, m8, stream))
        g88 = timed(lambda: qs.qs_sd4_linear_e4m3(x8, m8, w8, mw, b, M, N, K, out88, stream))
        same88 = bool(torch.equal(out.view(torch.int16), out88.view(torch.int16)))
        # the scales pre-arranged as the GEMM copies them (weights offline,
        # activations by one small pass per call): no block-word conversion
        # inside the GEMM
        xt = qs.sd4_scale_tiles(m8, False, stream=stream)
        wt = qs.sd4_scale_tiles(mw, True, stream=stream)
        out_t = torch.empty_like(out)
        qs.qs_sd4_linear_e4m3_tiles(x8, xt, w8, wt, b, M, N, K, out_t, stream)
        qt = timed(lambda: qs.qs_sd4_scale_tiles(m8, M, K, 0, xt, stream))
        gt = timed(lambda: qs.qs_sd4_linear_e4m3_tiles(x8, xt, w8, wt, b, M, N, K, out_t,
                                                       stream))
        same_t = bool(torch.equal(out.view(torch.int16), out_t.view(torch.int16)))
        # activation decomposition of the salient tokens (a seeded 1/16 of them)
        srows = I.salient_rows(M, cfg.seed)
        S_ = len(srows)
        rt = torch.tensor(srows, dtype=torch.int32, device=dev)
        c2 = torch.empty((S_, K), dtype=torch.uint8, device=dev)
        m2 = torch.empty((S_, K // 16), dtype=torch.int16, device=dev)
        out3 = out8.clone()
        for _ in range(warmup):
            qs.qs_sd4_quant_decomp(x, M, K, rt, S_, c2, m2, stream)
            qs.qs_sd4_linear_decomp(c2, m2, rt, S_, None, mw, w8, b, M, N, K, out3, stream)
        e3 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for e in e3:
            e[0].record(stream)
            qs.qs_sd4_quant_decomp(x, M, K, rt, S_, c2, m2, stream)
            e[1].record(stream)
            qs.qs_sd4_linear_decomp(c2, m2, rt, S_, None, mw, w8, b, M, N, K, out3, stream)
            e[2].record(stream)
        stream.synchronize()
        dq = sum(e[0].elapsed_time(e[1]) for e in e3) / steps
        dg = sum(e[1].elapsed_time(e[2]) for e in e3) / steps
        sel = rt[:rows].long()
        ref_s = x[sel].double() @ w.double().t() + b.double()
        err_s = lambda y: float((y - ref_s).norm() / ref_s.norm())  # noqa: E731
        decomp = {"salient_rows": S_, "salient_fraction": S_ / M, "quant_decomp_ms": dq,
                  "gemm_decomp_ms": dg,
                  "gemm_decomp_TFLOPS": 2.0 * S_ * 2 * K * N / (dg * 1e-3) / 1e12,
                  "layer_ms_e4m3_weights": q + g8 + dq + dg,
                  "rel_err_salient_plain": err_s(out8[sel].double()),
                  "rel_err_salient_decomposed": err_s(out3[sel].double()),
                  "error_rows": int(sel.numel())}
        ref = x[:rows].double() @ w.double().t() + b.double()
        wp, ws = qs.pack_weights(w, 4, stream=stream)
        xp, xs = qs.quant_act(x[:rows].contiguous(), 4, cfg.alpha, stream=stream)
        y4 = qs.qlinear(xp, xs, wp, ws, b, 4, K, stream=stream).double()
        stream.synchronize()
    err = lambda y: float((y - ref).norm() / ref.norm())  # noqa: E731
    pk, _ = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]  # measured bf16 x the nominal fp8:bf16 dense ratio
    tf = lambda ms: cfg.ops / (ms * 1e-3) / 1e12  # noqa: E731
    quant_bytes = M * (2 * K + K // 2 + 2 * (K // 32))
    return {"workload": cfg.name + "_sd4", "quant_ms": q,
            "gemm_ms": g, "gemm_path": "block-scaled fp8 (e4m3 + UE8M0 per 32), codes decoded",
            "TOPS": cfg.ops / ((q + g) * 1e-3) / 1e12, "gemm_TFLOPS": tf(g),
            "gemm_frac_fp8_peak": tf(g) / fp8_peak,
            "gemm_e4m3_weights_ms": g8, "gemm_e4m3_weights_TFLOPS": tf(g8),
            "gemm_e4m3_weights_frac_fp8_peak": tf(g8) / fp8_peak,
            "e4m3_weights_output_identical": same,
            "quant_e4m3_ms": q8, "gemm_e4m3_both_ms": g88, "gemm_e4m3_both_TFLOPS": tf(g88),
            "gemm_e4m3_both_frac_fp8_peak": tf(g88) / fp8_peak,
            "e4m3_both_output_identical": same88,
            "layer_e4m3_ms": q8 + g88, "layer_e4m3_TOPS": cfg.ops / ((q8 + g88) * 1e-3) / 1e12,
            "scale_tiles_ms": qt, "gemm_e4m3_tiles_ms": gt, "gemm_e4m3_tiles_TFLOPS": tf(gt),
            "gemm_e4m3_tiles_frac_fp8_peak": tf(gt) / fp8_peak,
            "e4m3_tiles_output_identical": same_t,
            "layer_e4m3_tiles_ms": q8 + qt + gt,
            "layer_e4m3_tiles_TOPS": cfg.ops / ((q8 + qt + gt) * 1e-3) / 1e12,
            "gemm_bf16_weights_ms": g2, "gemm_bf16_weights_TFLOPS": tf(g2),
            "gemm_bf16_weights_frac_bf16_peak": tf(g2) / pk["bf16_tflops"],
            "quant_GBps": quant_bytes / (q * 1e-3) / 1e9,
            "rel_err_sd4": err(out[:rows].double()), "rel_err_w4a4_rotated": err(y4),
            "error_rows": rows, "decomposition": decomp}


def quality(qs, torch, x, w, bias, bits, alpha, stream, rows=256):
    """Relative Frobenius error and SQNR of the layer against the unquantised
    binary64 product, with and without the Hadamard rotation (first `rows` tokens)."""
    xs_, ws_, b = x[:rows].contiguous(), w, bias
    ref = xs_.double() @ ws_.double().t() + b.double()
    out = {}
    for name, flags in (("rotated", 0), ("unrotated", qs.QS_FLAG_NO_ROTATE)):
        wp, wsc = qs.pack_weights(ws_, bits, flags, stream=stream)
        xp, xsc = qs.quant_act(xs_, bits, alpha, flags, stream=stream)
        y = qs.qlinear(xp, xsc, wp, wsc, b, bits, x.shape[1], stream=stream).double()
        stream.synchronize()
        err = (y - ref).norm() / ref.norm()
        out[name] = {"rel_fro_err": float(err), "sqnr_db": float(-20 * torch.log10(err))}
    return out


def run_reference(args, rank, world):
    """The CPU oracle timed as a bounded sample per step on every host core
    (rank 0 only; the other ranks exit without work)."""
    if rank != 0:
        return
    from bit_quantized_linear_hadamard_b200 import inputs as I
    cfg = workload_config(I, args.workload)
    rows_per_proc = 8
    d = I.make_layer(cfg, M=max(256, rows_per_proc * (os.cpu_count() or 1)))
    sample = OracleSample(d, cfg.bits, cfg.alpha, cfg.act_bits)
    pool = OraclePool(sample)
    try:
        for _ in range(args.warmup):
            pool.run(2)
        secs, rows = 0.0, 0
        for _ in range(args.steps):
            r, dt = pool.run(rows_per_proc)
            secs += dt
            rows += r
    finally:
        pool.close()
    value = 2.0 * rows * cfg.N * cfg.K / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4" if cfg.act_bits == cfg.bits == 4 else f"int{cfg.bits}w-int{cfg.act_bits}a",
        "data": "synthetic",
        "config": workload_line_config(cfg, args.act_codes, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": pool.procs, "kind": "oracle",
                         "host": host_info(),
                         "sample": f"{rows // args.steps} tokens per step ({rows_per_proc} per "
                                   f"process, one numpy process per host core) of the "
                                   f"{cfg.M}-token workload, full K and N"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    import bit_quantized_linear_hadamard_b200 as qs
    from bit_quantized_linear_hadamard_b200 import inputs as I

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    qs.load()

    cfg = workload_config(I, args.workload)
    d = I.make_layer(cfg, M=args.tokens)
    M, K, N, alpha = d["x"].shape[0], cfg.K, cfg.N, cfg.alpha
    bits, bx = cfg.bits, cfg.act_bits  # weight and activation code widths
    x_flags = qs.QS_FLAG_BYTE_CODES if (args.act_codes == "bytes" and bx == 4) else 0
    sx = qs.storage_bits(bx, x_flags)  # storage width the GEMM reads
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        x = d["x"].to(dev)
        w = d["w"].to(dev)
        bias = d["bias"].to(dev)
        wp, ws = qs.pack_weights(w, bits, stream=stream)
        xp = torch.empty((M, qs.packed_cols(K, bx, x_flags)), dtype=torch.uint8, device=dev)
        xs = torch.empty((M,), dtype=torch.float32, device=dev)
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    stream.synchronize()
    del w

    def gemm():
        if sx == bits:
            qs.qs_qlinear(xp, xs, wp, ws, bias, M, N, K, bits, out, stream)
        else:
            qs.qs_qlinear_mixed(xp, xs, sx, wp, ws, bits, bias, M, N, K, out, stream)

    def step():
        qs.qs_quant_act(x, M, K, bx, alpha, x_flags, xp, xs, stream)
        gemm()

    for _ in range(max(3, args.warmup)):
        step()
    stream.synchronize()
    if qs.qs_device_error(stream) != 0:
        raise SystemExit("kernel wait timed out during warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
        sampler.mark_start()
    for i in range(args.steps):
        ev[i][0].record(stream)
        qs.qs_quant_act(x, M, K, bx, alpha, x_flags, xp, xs, stream)
        ev[i][1].record(stream)
        gemm()
        ev[i][2].record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_end()
    clocks = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()
    total_ms = ev[0][0].elapsed_time(ev[-1][2])
    quant_each = [e[0].elapsed_time(e[1]) for e in ev]
    gemm_each = [e[1].elapsed_time(e[2]) for e in ev]
    quant_ms = sum(quant_each) / args.steps
    gemm_ms = sum(gemm_each) / args.steps
    if qs.qs_device_error(stream) != 0:
        raise SystemExit("kernel wait timed out in the timed region")

    ops_per_step = 2.0 * M * N * K
    comb = combine_ranks([total_ms, quant_ms, gemm_ms], args.steps, ops_per_step, world, dev)
    total_ms, quant_ms, gemm_ms = comb["times_ms"]
    ms_per_step, value = comb["ms_per_step"], comb["value"]

    ref_rows = out[::1009].clone()  # the device step's output, to check the end-to-end one
    quant_alone_ms = combine_ranks([time_quant_alone(qs, torch, x, bx, alpha, x_flags, stream)],
                                   1, ops_per_step, world, dev)["times_ms"][0]
    # ---- end to end through the same C ABI calls, inputs and result in pinned host memory
    x_host = d["x"].pin_memory()
    out_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(1, args.e2e_steps)

    # chunks of tokens: chunk i's layer call (one public C call, qs_linear_ex)
    # runs while chunk i+1 is copied in and chunk i-1 copied out
    n_chunks = max(1, min(args.e2e_chunks, M))
    rows_per = (M + n_chunks - 1) // n_chunks
    spans = [(r0, min(M, r0 + rows_per)) for r0 in range(0, M, rows_per)]
    ws_bytes = qs.qs_linear_workspace_bytes(rows_per, K, sx)
    workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    copied_out = [None] * len(spans)  # per chunk: the last copy-out of its output rows

    def e2e_step():
        for i, (r0, r1) in enumerate(spans):
            with torch.cuda.stream(s_in):
                x[r0:r1].copy_(x_host[r0:r1], non_blocking=True)
                got = torch.cuda.Event()
                got.record(s_in)
            stream.wait_event(got)
            if copied_out[i] is not None:  # the previous step's rows have left the device
                stream.wait_event(copied_out[i])
            qs.qs_linear_ex(x[r0:r1], r1 - r0, K, alpha, bx, x_flags, wp, ws, bits, bias, N,
                            workspace, ws_bytes, out[r0:r1], stream)
            done = torch.cuda.Event()
            done.record(stream)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                out_host[r0:r1].copy_(out[r0:r1], non_blocking=True)
                copied_out[i] = torch.cuda.Event()
                copied_out[i].record(s_out)
        # the next step's copies overwrite x: they wait for this step's layer calls
        fin = torch.cuda.Event()
        fin.record(stream)
        s_in.wait_event(fin)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for _ in range(e2e_steps):
        e2e_step()
    last = torch.cuda.Event()
    last.record(s_out)
    s_in.wait_event(last)   # e1 follows every copy, layer call and copy-out
    e1.record(s_in)
    torch.cuda.synchronize()
    e2e_ms = combine_ranks([e0.elapsed_time(e1) / e2e_steps], 1, ops_per_step, world,
                           dev)["times_ms"][0]
    e2e_same = bool(torch.equal(out_host[::1009].to(dev).view(torch.int16),
                                ref_rows.view(torch.int16)))

    # both storages of 4-bit activation codes, timed the same way (the
    # headline's own numbers are the ones measured above)
    layouts = {}
    if bx == 4:
        for name, flags in (("packed", 0), ("bytes", qs.QS_FLAG_BYTE_CODES)):
            if flags == x_flags:
                q_ms, g_ms = quant_ms, gemm_ms
            else:
                q_ms, g_ms, _ = time_layer(qs, torch, x, wp, ws, bias, bits, alpha, stream,
                                           steps=args.steps, warmup=3, bits_x=bx, x_flags=flags)
                q_ms, g_ms = combine_ranks([q_ms, g_ms], 1, ops_per_step, world, dev)["times_ms"]
            layouts[name] = {"quant_ms": q_ms, "gemm_ms": g_ms, "step_ms": q_ms + g_ms,
                             "x_flags": flags, "headline": flags == x_flags}

    extra = {}
    if world == 1 and not args.no_extras:
        if bx == bits:
            extra["quality"] = quality(qs, torch, x, d["w"].to(dev), bias, bits, alpha, stream)
        extra["configs"] = all_configs(qs, torch, I, dev, stream)
        extra["gbs"] = gbs_sequence(qs, torch, I, dev, stream)
        extra["bgr"] = bgr_layer(qs, torch, I, dev, stream)
        extra["sd4"] = sd4_layer(qs, torch, I, dev, stream)
    if rank == 0:
        pk, src = peaks()
        int8_peak = pk["bf16_tflops"] * INT8_PER_BF16
        gemm_tops = ops_per_step / (gemm_ms * 1e-3) / 1e12
        # algorithmic bytes of the activation kernel per token: read 2K (bf16),
        # write K*b/8 (codes at their width b) and 4 (scale), whatever the
        # storage layout; the bytes a layout actually writes are reported beside
        quant_bytes = M * (2 * K + K * bx // 8 + 4)
        stored_bytes = M * (2 * K + qs.packed_cols(K, bx, x_flags) + 4)
        traffic_key = cfg.name + ("_act_codes_in_bytes" if x_flags else "")
        headline_fam, headline_inst = gemm_kernel(4 if sx == 4 else 8, 4 if bits == 4 else 8)
        quant_gbs = quant_bytes / (quant_ms * 1e-3) / 1e9
        for name, L in layouts.items():
            key = cfg.name + ("_act_codes_in_bytes" if L["x_flags"] else "")
            g_tops = ops_per_step / (L["gemm_ms"] * 1e-3) / 1e12
            q_gbs = quant_bytes / (L["quant_ms"] * 1e-3) / 1e9
            fam, inst = gemm_kernel(8 if L["x_flags"] else 4, 4 if bits == 4 else 8)
            L.update({
                "TOPS": ops_per_step * world / (L["step_ms"] * 1e-3) / 1e12,
                "tokens_per_s": M * world / (L["step_ms"] * 1e-3),
                "gemm_TOPS": g_tops, "gemm_frac_int8_peak": g_tops / int8_peak,
                "gemm_kernel": inst,
                "gemm_traffic": ncu_traffic(key, fam),
                "quant_GBps": q_gbs, "quant_frac_hbm": q_gbs / pk["hbm_gbs"],
                "quant_stored_bytes": M * (2 * K + qs.packed_cols(K, bx, L["x_flags"]) + 4),
                "quant_traffic": ncu_traffic(key, "rotate_quant_kernel")})
        line = {
            "metric": METRIC, "value": value, "unit": UNIT,
            "tokens_per_s": M * world / (ms_per_step * 1e-3),
            "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "data": "synthetic",
            "dtype": "int4" if bx == bits == 4 else f"int{bits}w-int{bx}a",
            "config": workload_line_config(cfg, "bytes" if x_flags else "packed", world, M=M),
            "roofline": {"bound": "tensor", "achieved": gemm_tops, "peak": int8_peak,
                         "unit": UNIT, "frac": gemm_tops / int8_peak,
                         "traffic": ncu_traffic(traffic_key, headline_fam),
                         "kernel": headline_inst,
                         "peak_source": f"{src}: bf16_tflops (burst) x {INT8_PER_BF16} "
                                        f"nominal int8:bf16"},
            "roofline_quant": {"bound": "hbm", "achieved": quant_gbs, "peak": pk["hbm_gbs"],
                               "unit": "GB/s", "frac": quant_gbs / pk["hbm_gbs"],
                               "traffic": ncu_traffic(traffic_key, "rotate_quant_kernel"),
                               "algorithmic_bytes": quant_bytes,
                               "algorithmic_bytes_rule": "M*(2K + K*b/8 + 4), b the code width",
                               "stored_bytes": stored_bytes,
                               "peak_source": f"{src}: hbm_gbs",
                               "alone": {
                                   "ms": quant_alone_ms,
                                   "achieved": quant_bytes / (quant_alone_ms * 1e-3) / 1e9,
                                   "frac": quant_bytes / (quant_alone_ms * 1e-3) / 1e9
                                           / pk["hbm_gbs"],
                                   "note": "the same kernel launched back to back on its own; "
                                           "in the step it follows the GEMM, whose last output "
                                           "lines are written back from L2 while it runs"}},
            "act_code_layouts": layouts,
            "kernels_ms": {"quant": quant_ms, "gemm": gemm_ms},
            "kernels_ms_median": {"quant": statistics.median(quant_each),
                                  "gemm": statistics.median(gemm_each)},
            "gpu_launches": 2 * args.steps,
            "e2e": {"value": ops_per_step * world / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": x_host.numel() * 2,
                    "d2h_bytes_per_step": out_host.numel() * 2,
                    "ms_per_step": e2e_ms, "steps": e2e_steps,
                    "call": "qs_linear_ex (C ABI: activation kernel + GEMM) per token chunk, pinned "
                            "host x in, bf16 output back, copies overlapped with the layer",
            "chunks": n_chunks, "output_equals_device_step": e2e_same},
            "clocks": clocks,
        }
        line.update(extra)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = OracleSample(d, bits, alpha, bx).baseline()
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
