"""Benchmark of the SRU layer on B200.

One step = one pass of the whole hot path over one batch: the projection
U = X W_cat^T (tcgen05 GEMM), the forward recurrence, the backward recurrence
(+ the dv/db reduction), and the projection gradients dX += dU W_cat and
dW_cat = dU^T X.  Workload: the language-model training layer, L = 1024,
B = 16 tokens-per-step rows, d = 2048, bf16 projection and fp32 recurrence
(seeded synthetic inputs; no dataset).

Prints ONE JSON line (rank 0).  `value` is device-timed throughput (tokens/s)
with inputs resident in HBM; `e2e` is the same step through the same C-ABI
calls with the per-step inputs copied from pinned host memory and every
gradient (dx, dW, dv, db, dc0) copied back inside the timed region.
`workloads` holds device-timed results of every other layer workload (the
forward-only layer, the bidirectional masked layer, the recurrence-only layer
with v != 0 and v = 0, and a layer in the chunked scan's regime), each kernel
against its roofline.  The tensor-core peak is chosen from the clock samples
taken while the kernels ran: the burst figure when the SM clock stayed within
5 % of its maximum with no power-cap sample, the sustained one otherwise.

--impl reference times the fp64 CPU oracle (the baseline the library is
checked against) on the host cores, on a bounded sample per step, and
extrapolates to the full step (said so in its line).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SRU fwd+bwd tokens/s and recurrence HBM GB/s (% of peak) on 1 B200"
WORKLOAD = "lm_train"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            pk = json.load(fh)
        return dict(hbm_gbs=float(pk["hbm_gbs"]), bf16_tflops=float(pk["bf16_tflops"]),
                    bf16_tflops_sustained=float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0


def tensor_peak(peaks, clocks):
    """The bf16 peak that applies to kernels run under these sampled clocks:
    the burst figure (cuBLAS timed alone at full clock) when the median SM clock
    stayed within 5 % of its maximum and no sample saw the power cap, else the
    sustained figure (a seconds-long loop under the power cap)."""
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    burst = (sm is not None and mx and sm >= 0.95 * mx and "sw_power_cap" not in clocks.get("reasons", []))
    if burst:
        return "burst", peaks["bf16_tflops"]
    return "sustained", peaks["bf16_tflops_sustained"]


SRC_DIRS = (os.path.join(ROOT, "parallelizable_recurrence_b200", "csrc"), os.path.join(ROOT, "include"))
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")


def library_source_hash() -> str:
    """sha256 over the library's CUDA/C sources (file names and contents, sorted)."""
    import hashlib
    h = hashlib.sha256()
    for d in SRC_DIRS:
        for name in sorted(os.listdir(d)):
            if name.endswith((".cu", ".cuh", ".h")):
                h.update(name.encode())
                with open(os.path.join(d, name), "rb") as fh:
                    h.update(fh.read())
    return h.hexdigest()


def load_traffic():
    """ncu DRAM bytes (read + write) per launch, keyed by workload and phase, from
    the capture recorded beside the profiles -- only if that capture was taken of
    these exact library sources (same hash); otherwise {} and traffic is null."""
    if not os.path.exists(TRAFFIC_FILE):
        return {}, "no ncu capture recorded"
    with open(TRAFFIC_FILE) as fh:
        rec = json.load(fh)
    if rec.get("source_hash") != library_source_hash():
        return {}, "ncu capture was of other library sources (stale): traffic not reported"
    return rec.get("bytes_per_launch", {}), rec.get("command", "")


def host_info():
    model = None
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def workload_config():
    from synthetic import CONFIGS
    cfg = CONFIGS[WORKLOAD]
    return cfg, {"workload": f"{cfg.name}: SRU layer training step L={cfg.L} B={cfg.B} d={cfg.d} "
                             f"unidirectional, bf16 projection, fp32 recurrence",
                 "L": cfg.L, "B_per_gpu": cfg.B, "d": cfg.d, "tokens_per_step_per_gpu": cfg.tokens,
                 "l2": "inputs larger than L2 (step working set ~1.3 GB vs 126 MB L2); no flush"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons every few
    milliseconds through NVML while the timed region runs (nvidia-smi as a
    fallback when NVML is unavailable).  Reads only; changes no setting."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index = index
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self._nvml = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self._nvml = (pynvml, h)
        except Exception:
            self._nvml = None
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                self._sample()
                self._stop.wait(self.period)
        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def _sample(self):
        if self._nvml is not None:
            pynvml, h = self._nvml
            try:
                self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.reasons.update(n for b, n in self.REASONS.items() if bits & b)
            except Exception:
                pass
            return
        try:
            out = subprocess.run(["nvidia-smi", "-i", str(self.index), "--query-gpu=clocks.sm,clocks.max.sm,"
                                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                                  "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5).stdout
            parts = [p.strip() for p in out.split(",")]
            self.samples.append(float(parts[0]))
            self.max_mhz = float(parts[1])
            for n, v in zip(["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"], parts[2:]):
                if v.lower() == "active":
                    self.reasons.add(n)
        except Exception:
            pass

    def __exit__(self, *a):
        self._stop.set()
        self._thread.join(timeout=5)
        if not self.samples:
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "nvml" if self._nvml is not None else "nvidia-smi"}


# ---------------------------------------------------------- CPU baseline
def cpu_baseline(cfg, budget_s: float = 10.0, seed: int = 0):
    """Time the fp64 oracle on a bounded sample of the workload on one host core
    and extrapolate to the full step (projection, its two gradients, forward and
    backward recurrence over every channel).  Returns (tokens/s, description,
    extrapolated seconds per full step, seconds of oracle work measured)."""
    import oracle
    from synthetic import f32_to_bf16_bits
    rng = np.random.default_rng(seed)
    L, B, d = cfg.L, cfg.B, cfg.d
    M, N, K = L * B, cfg.N, d
    # recurrence: every batch row of n_ch channels, all L steps
    n_ch = 8
    U = rng.standard_normal((L, B, 1, 3, n_ch))
    x = rng.standard_normal((L, B, n_ch))
    v = rng.uniform(-0.5, 0.5, (1, 2, n_ch))
    bias = 0.1 * rng.standard_normal((1, 2, n_ch))
    dh = rng.standard_normal((L, B, 1, n_ch))
    t_start = t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.forward(U, x, v, bias)
        oracle.backward(U, x, v, bias, dh)
        reps += 1
        if time.perf_counter() - t0 > budget_s * 0.3:
            break
    t_rec = (time.perf_counter() - t0) / (reps * B * n_ch)          # s per channel (fwd + bwd)
    # projection and gradients: entries of each product, each a K_red-long plain sum
    Xb = f32_to_bf16_bits(rng.standard_normal((512, K)).astype(np.float32))
    Wb = f32_to_bf16_bits(rng.standard_normal((512, K)).astype(np.float32))
    rows = rng.integers(0, 512, 64)
    cols = rng.integers(0, 512, 64)
    t0 = time.perf_counter()
    n_ent = 0
    while True:
        oracle.project_entries(Xb, Wb, rows, cols)
        n_ent += rows.size
        if time.perf_counter() - t0 > budget_s * 0.7:
            break
    t_mac = (time.perf_counter() - t0) / (n_ent * K)                # s per multiply-add
    measured = time.perf_counter() - t_start
    full = t_rec * B * d * cfg.n_dir + t_mac * 3 * M * N * K
    desc = (f"fp64 oracle, 1 thread: recurrence fwd+bwd on {n_ch} channels x {B} rows x L={L} "
            f"({reps} reps), projection plain sums {n_ent} entries x K={K}, {measured:.1f} s measured; "
            f"extrapolated to the full step ({B * d * cfg.n_dir} channels, 3 products of {M}x{N}x{K})")
    return cfg.tokens / full, desc, full, measured


# ------------------------------------------------------ per-workload block
def _time_ms(fn, flush, reps=10, warm=3):
    """Median device time (ms) of fn() on torch's current stream, CUDA events,
    after `warm` untimed calls; `flush` (a buffer larger than L2) is rewritten
    before every timed call so that no input is served from L2."""
    import torch
    st = torch.cuda.current_stream()
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        fn()
        b.record(st)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return float(statistics.median(ts))


def _lengths(L, B, seed):
    """Sequence lengths of a padded batch: integers uniform on [L/2, L]."""
    return np.random.default_rng(seed).integers(L // 2, L, size=B, endpoint=True)


def _hbm_entry(kernel, ms, nbytes):
    return {"kernel": kernel, "bound": "hbm", "ms": ms, "algorithmic_bytes": nbytes,
            "achieved": nbytes / (ms / 1e3) / 1e9, "unit": "GB/s"}


def _tc_entry(kernel, ms, flops):
    return {"kernel": kernel, "bound": "tensor", "ms": ms, "algorithmic_flops": flops,
            "achieved": flops / (ms / 1e3) / 1e12, "unit": "TFLOP/s"}


class _Layer:
    """Device buffers of one layer workload, drawn on the device from a seeded
    generator with the workload's distributions (U or X and W, x, v, b, c0, dh,
    padding lengths)."""

    def __init__(self, L, B, d, nd, seed, dev, masked=False, v_zero=False, project=False, c0=False):
        import torch
        import parallelizable_recurrence_b200 as sru
        self.L, self.B, self.d, self.nd = L, B, d, nd
        g = torch.Generator(device=dev).manual_seed(seed)
        self.x = torch.randn(L, B, d, device=dev, generator=g)
        if project:
            a = (3.0 / d) ** 0.5
            self.X = self.x.view(L * B, d).to(torch.bfloat16)
            self.W = ((torch.rand(nd * 3 * d, d, device=dev, generator=g) * 2 - 1) * a).to(torch.bfloat16)
        self.U = torch.randn(L, B, nd, 3, d, device=dev, generator=g).to(torch.bfloat16)
        self.v = torch.zeros(nd, 2, d, device=dev) if v_zero else torch.rand(nd, 2, d, device=dev, generator=g) - 0.5
        self.b = 0.1 * torch.randn(nd, 2, d, device=dev, generator=g)
        self.c0 = torch.randn(B, nd, d, device=dev, generator=g) if c0 else None
        self.dh = torch.randn(L, B, nd, d, device=dev, generator=g)
        self.mask = None
        self.valid = 1.0
        if masked:
            lengths = _lengths(L, B, seed)
            m = (np.arange(L)[:, None] >= lengths[None, :]).astype(np.uint8)
            self.mask = torch.from_numpy(m).to(dev)
            self.valid = float((m == 0).mean())
        self.h = torch.empty(L, B, nd, d, device=dev)
        self.cT = torch.empty(B, nd, d, device=dev)
        self.dU = torch.empty(L, B, nd, 3, d, device=dev, dtype=torch.bfloat16)
        self.dx = torch.empty(L, B, d, device=dev)
        self.dv = torch.empty(nd, 2, d, device=dev)
        self.db = torch.empty(nd, 2, d, device=dev)
        self.dc0 = torch.empty(B, nd, d, device=dev)
        flags = (sru.SRU_FLAG_V_ZERO | sru.SRU_FLAG_FORCE_SCAN) if v_zero else sru.SRU_FLAG_FORCE_SCAN
        self.ws = sru.alloc_workspace(L, B, d, nd == 2, flags, device=dev)

    @property
    def elements(self):
        return self.L * self.B * self.d * self.nd

    def fwd_bytes(self):
        """U 6 + x 4 + h 4 bytes per valid element; h (zeros) 4 per padded one."""
        e = self.elements
        return 14.0 * e * self.valid + 4.0 * e * (1 - self.valid)

    def bwd_bytes(self):
        """U 6 + x 4 + dh 4 + dU 6 + dx 4 bytes per valid element; per padded one the
        zero dU (6) and, once per position for both directions, the zero dx (4)."""
        e = self.elements
        return 24.0 * e * self.valid + (6.0 + 4.0 / self.nd) * e * (1 - self.valid)

    def forward(self, flags=0):
        import parallelizable_recurrence_b200 as sru
        sru.sru_forward(self.U, self.x, self.v, self.b, self.h, self.cT, c0=self.c0, mask=self.mask,
                        bidirectional=self.nd == 2, flags=flags, workspace=self.ws)

    def backward(self, flags=0):
        import parallelizable_recurrence_b200 as sru
        sru.sru_backward(self.U, self.x, self.v, self.b, self.dh, self.ws, self.dU, self.dx, self.dv, self.db,
                         self.dc0, c0=self.c0, mask=self.mask, bidirectional=self.nd == 2, flags=flags)


def _recurrence_entries(lay, flush, variants, tag=""):
    out = {}
    for name, fl in variants:
        tf = _time_ms(lambda: lay.forward(fl), flush)
        lay.forward(fl)  # the backward reads this variant's checkpoints
        tb = _time_ms(lambda: lay.backward(fl), flush)
        out[f"forward{tag}{name}"] = _hbm_entry("sru_forward", tf, lay.fwd_bytes())
        out[f"backward{tag}{name}"] = _hbm_entry("sru_backward", tb, lay.bwd_bytes())
    return out


def _gemm_entries(lay, flush):
    import torch
    import parallelizable_recurrence_b200 as sru
    M, N, K = lay.L * lay.B, lay.nd * 3 * lay.d, lay.d
    fl = 2.0 * M * N * K
    Uv = lay.U.view(M, N)
    dX = torch.empty(M, K, device=lay.x.device)
    dW = torch.empty(N, K, device=lay.x.device)
    dUv = lay.dU.view(M, N).copy_(Uv)
    t_u = _time_ms(lambda: sru.sru_project(lay.X, lay.W, Uv), flush)
    t_dx = _time_ms(lambda: sru.sru_project_backward(dUv, lay.X, lay.W, dX=dX, accumulate=True), flush)
    t_dw = _time_ms(lambda: sru.sru_project_backward(dUv, lay.X, lay.W, dW=dW), flush)
    return {"project": _tc_entry("sru_project (U = X W^T)", t_u, fl),
            "project_dX": _tc_entry("sru_project_backward (dX += dU W)", t_dx, fl),
            "project_dW": _tc_entry("sru_project_backward (dW = dU^T X)", t_dw, fl)}


def _fused_entry(lay, ms, with_u):
    """The fused forward against the roofline of a kernel that is both a product
    and a stream: its time bound is the larger of flops / tensor peak and
    algorithmic bytes / HBM peak (bytes: X 2 B per (t, b, k), W_cat once, x 4 and
    h 4 per element, + U 6 per element when it is stored)."""
    L, B, d, nd = lay.L, lay.B, lay.d, lay.nd
    flops = 2.0 * L * B * nd * 3 * d * d
    nbytes = 2.0 * L * B * d + 2.0 * nd * 3 * d * d + (4.0 + (6.0 if with_u else 0.0)) * lay.elements + 4.0 * L * B * d
    return {"kernel": "sru_forward_fused" + (" (U stored)" if with_u else " (inference: no U)"), "bound": "mixed",
            "ms": ms, "algorithmic_flops": flops, "algorithmic_bytes": nbytes,
            "achieved_tflops": flops / (ms / 1e3) / 1e12, "achieved_gbs": nbytes / (ms / 1e3) / 1e9,
            "tokens_per_s": L * B / (ms / 1e3)}


def _layer_rec_only(dev, flush, sru):
    lay = _Layer(1024, 16, 3072, 1, 4, dev)
    out = {"rec_only L1024 B16 d3072 v!=0": _recurrence_entries(lay, flush, [("", 0)])}
    lay.v.zero_()
    VZ, SCAN, SEQ = sru.SRU_FLAG_V_ZERO, sru.SRU_FLAG_FORCE_SCAN, sru.SRU_FLAG_FORCE_SEQUENTIAL
    out["rec_only_v0 L1024 B16 d3072 v=0"] = _recurrence_entries(
        lay, flush, [("_dispatched", VZ), ("_scan_forced", VZ | SCAN), ("_sequential_forced", VZ | SEQ)])
    return out


def _layer_scan_regime(dev, flush, sru):
    # a layer in the chunked scan's regime (B*d too small to fill the GPU), v = 0
    lay = _Layer(2048, 4, 2048, 1, 5, dev, v_zero=True)
    VZ, SEQ = sru.SRU_FLAG_V_ZERO, sru.SRU_FLAG_FORCE_SEQUENTIAL
    return {"scan_regime L2048 B4 d2048 v=0": _recurrence_entries(
        lay, flush, [("_dispatched", VZ), ("_sequential_forced", VZ | SEQ)])}


def _layer_lm_fwd(dev, flush, sru):
    # forward-only language-model layer, bf16 projection
    L, B, d = 256, 32, 512
    lay = _Layer(L, B, d, 1, 1, dev, project=True)
    e = {"project": _gemm_entries(lay, flush)["project"]}
    e["forward"] = _hbm_entry("sru_forward", _time_ms(lambda: lay.forward(0), flush), lay.fwd_bytes())
    t_step = _time_ms(lambda: (sru.sru_project(lay.X, lay.W, lay.U.view(L * B, 3 * d)), lay.forward(0)), flush)
    e["layer_two_calls"] = {"ms": t_step, "tokens_per_s": L * B / (t_step / 1e3), "calls": "sru_project + sru_forward"}
    t_f = _time_ms(lambda: sru.sru_forward_fused(lay.X, lay.W, lay.x, lay.v, lay.b, lay.h, lay.cT, lay.ws), flush)
    e["layer_fused"] = _fused_entry(lay, t_f, with_u=False)
    return {"lm_fwd L256 B32 d512 forward": e}


def _layer_lm_train_fused(dev, flush, sru):
    # the training layer's forward: two calls vs fused (U and checkpoints stored for the backward)
    L, B, d = 1024, 16, 2048
    lay = _Layer(L, B, d, 1, 2, dev, project=True, c0=True)
    t2 = _time_ms(lambda: (sru.sru_project(lay.X, lay.W, lay.U.view(L * B, 3 * d)), lay.forward(0)), flush)
    t_f = _time_ms(lambda: sru.sru_forward_fused(lay.X, lay.W, lay.x, lay.v, lay.b, lay.h, lay.cT, lay.ws,
                                                 c0=lay.c0, U=lay.U), flush)
    t_i = _time_ms(lambda: sru.sru_forward_fused(lay.X, lay.W, lay.x, lay.v, lay.b, lay.h, lay.cT, lay.ws,
                                                 c0=lay.c0), flush)
    return {"lm_train L1024 B16 d2048 forward": {
        "layer_two_calls": {"ms": t2, "tokens_per_s": L * B / (t2 / 1e3), "calls": "sru_project + sru_forward"},
        "layer_fused_with_U": _fused_entry(lay, t_f, with_u=True),
        "layer_fused_inference": _fused_entry(lay, t_i, with_u=False)}}


def _layer_bidir(dev, flush, sru):
    # bidirectional padded layer, 2 directions
    lay = _Layer(2048, 64, 1024, 2, 3, dev, masked=True, project=True)
    # the latency-bound recurrences first, before the products draw the power cap
    e = _recurrence_entries(lay, flush, [("", 0)], tag="_masked")
    e["valid_fraction"] = lay.valid
    mask = lay.mask
    lay.mask, lay.valid = None, 1.0
    e.update(_recurrence_entries(lay, flush, [("", 0)], tag="_unmasked"))
    lay.mask = mask
    e.update(_gemm_entries(lay, flush))
    t_f = _time_ms(lambda: sru.sru_forward_fused(lay.X, lay.W, lay.x, lay.v, lay.b, lay.h, lay.cT, lay.ws,
                                                 mask=lay.mask, bidirectional=True, U=lay.U), flush)
    e["layer_fused_with_U_masked"] = _fused_entry(lay, t_f, with_u=True)
    return {"bidir_masked L2048 B64 d1024 x2": e}


def _layer_producers(dev, flush, sru):
    # the other producers of U at the training layer's shape (d' = d/4): the factorised
    # projection (forward and backward) and SRU++'s attention producer
    import torch
    L, B, d = 1024, 16, 2048
    dp, M, N = d // 4, L * B, 3 * d
    g = torch.Generator(device=dev).manual_seed(6)
    X = torch.randn(M, d, device=dev, generator=g).to(torch.bfloat16)
    Wq = ((torch.rand(dp, d, device=dev, generator=g) * 2 - 1) * (3.0 / d) ** 0.5).to(torch.bfloat16)
    Wo = ((torch.rand(N, dp, device=dev, generator=g) * 2 - 1) * (3.0 / dp) ** 0.5).to(torch.bfloat16)
    Wkv = ((torch.rand(2 * dp, dp, device=dev, generator=g) * 2 - 1) * (3.0 / dp) ** 0.5).to(torch.bfloat16)
    P = torch.empty(M, dp, device=dev, dtype=torch.bfloat16)
    U = torch.empty(M, N, device=dev, dtype=torch.bfloat16)
    dU = torch.randn(M, N, device=dev, generator=g).to(torch.bfloat16)
    dP = torch.empty(M, dp, device=dev, dtype=torch.bfloat16)
    dX = torch.zeros(M, d, device=dev)
    dWq, dWo = torch.empty(dp, d, device=dev), torch.empty(N, dp, device=dev)
    ffl = 2.0 * M * dp * (d + N)
    t_f = _time_ms(lambda: sru.sru_project_factored(X, Wq, Wo, P, U), flush)
    t_fb = _time_ms(lambda: sru.sru_project_factored_backward(dU, X, Wq, Wo, P, dP, dX=dX, accumulate=True,
                                                              dWq=dWq, dWo=dWo), flush)
    aws = torch.empty(int(sru.load_library().sru_attention_workspace_bytes(L, B, dp)), dtype=torch.uint8,
                      device=dev)
    proj = 2.0 * M * dp * (d + 2 * dp + N)  # Q, [K | V] and the output products
    e = {"factored": _tc_entry("sru_project_factored (U = (X Wq^T) Wo^T)", t_f, ffl),
         "factored_backward": _tc_entry("sru_project_factored_backward (dX, dWq, dWo)", t_fb, 2.0 * ffl)}
    for causal in (True, False):
        # scores and P.V: 2 L^2 d' flops each per batch row, or only the (t, s <= t) entries when causal
        att = 2.0 * 2.0 * B * dp * (L * (L + 1) / 2.0 if causal else float(L * L))
        t_a = _time_ms(lambda: sru.sru_attention_project(X, Wq, Wkv, Wo, U, L, B, 0.5, causal=causal,
                                                         workspace=aws), flush)
        ent = _tc_entry("sru_attention_project (" + ("causal" if causal else "full") + " attention)", t_a,
                        proj + att)
        ent["tokens_per_s"] = M / (t_a / 1e3)
        e["attention_causal" if causal else "attention_full"] = ent
    # the producer's backward (causal, with the norm): the gradients of the four
    # projections (two products each) and of the attention (dP, dV, dK, dQ: four
    # products of the scores' size); the recomputation of the scores is not counted
    bws = torch.empty(int(sru.load_library().sru_attention_backward_workspace_bytes(L, B, d, dp, N)),
                      dtype=torch.uint8, device=dev)
    gam, bet = torch.ones(dp, device=dev), torch.zeros(dp, device=dev)
    dgam, dbet = torch.empty(dp, device=dev), torch.empty(dp, device=dev)
    dWkv = torch.empty(2 * dp, dp, device=dev)
    sru.sru_attention_project(X, Wq, Wkv, Wo, U, L, B, 0.5, ln_gamma=gam, ln_beta=bet, workspace=aws)
    t_ab = _time_ms(lambda: sru.sru_attention_project_backward(dU, X, Wq, Wkv, Wo, L, B, 0.5, aws, dX, dWq, dWkv, dWo,
                                                               ln_gamma=gam, ln_beta=bet, dgamma=dgam, dbeta=dbet,
                                                               workspace=bws), flush)
    ent = _tc_entry("sru_attention_project_backward (causal, layer norm)", t_ab,
                    2.0 * proj + 4.0 * 2.0 * B * dp * (L * (L + 1) / 2.0))
    ent["tokens_per_s"] = M / (t_ab / 1e3)
    e["attention_backward_causal"] = ent
    return {"producers L1024 B16 d2048 d'512": e}


# recurrence-only layers first, the product-heavy ones last (so that a power
# cap reached under the products does not slow the latency-bound recurrences)
WORKLOAD_LAYERS = {"rec_only": _layer_rec_only, "scan_regime": _layer_scan_regime, "lm_fwd": _layer_lm_fwd,
                   "lm_train_fused": _layer_lm_train_fused, "producers": _layer_producers, "bidir_masked": _layer_bidir}


def measure_workloads(dev, peaks, only=None):
    """Device-timed kernels of the other layer workloads, each alone with L2
    flushed before every timed call (median of 10 after 3 warm-up calls).  The
    clocks are sampled per layer and each layer's tensor peak chosen from them."""
    import torch
    import parallelizable_recurrence_b200 as sru
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    res, clocks_by_layer = {}, {}
    for key, fn in WORKLOAD_LAYERS.items():
        if only is not None and key != only:
            continue
        with ClockSampler(dev.index if dev.index is not None else 0, period_s=0.01) as clk:
            out = fn(dev, flush, sru)
            torch.cuda.synchronize()
        torch.cuda.empty_cache()
        clocks = clk.summary()
        kind, tc_peak = tensor_peak(peaks, clocks)
        for name, entries in out.items():
            clocks_by_layer[name] = dict(clocks, bf16_peak_kind=kind, bf16_peak=tc_peak)
            for ent in entries.values():
                if not isinstance(ent, dict) or "bound" not in ent:
                    continue
                if ent["bound"] == "hbm":
                    ent["peak"] = peaks["hbm_gbs"]
                    ent["frac"] = ent["achieved"] / peaks["hbm_gbs"]
                    ent["frac_of_nominal_8TBs"] = ent["achieved"] / NOMINAL_HBM_GBS
                elif ent["bound"] == "tensor":
                    ent["peak"] = tc_peak
                    ent["frac"] = ent["achieved"] / tc_peak
                    ent["frac_of_nominal_2250"] = ent["achieved"] / NOMINAL_BF16_TFLOPS
                else:  # a product and a stream: the larger of the two bounds
                    t_bound = max(ent["algorithmic_flops"] / (tc_peak * 1e12),
                                  ent["algorithmic_bytes"] / (peaks["hbm_gbs"] * 1e9))
                    ent["roofline_ms"] = t_bound * 1e3
                    ent["frac"] = t_bound / (ent["ms"] / 1e3)
            res[name] = entries
        time.sleep(0.5)  # let the power state settle before the next layer
    st = sru.sru_sync_status()
    if st != 0:
        raise RuntimeError(f"device status {st} in the workload block")
    return {"timing": "each kernel alone, median of 10 after 3 warm-up calls, 512 MB written before every "
                      "timed call (L2 flushed); inputs drawn on the device from seeded generators",
            "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_burst": peaks["bf16_tflops"],
                      "bf16_sustained": peaks["bf16_tflops_sustained"], "source": peaks["source"]},
            "clocks": clocks_by_layer, "layers": res}


# ------------------------------------------------------------ GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    import parallelizable_recurrence_b200 as sru
    from synthetic import generate

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    sru.load_library()
    peaks = load_peaks()
    cfg, config = workload_config()
    cfg = cfg.replace(seed=cfg.seed + 100 * rank)      # each rank its own batch (data parallel)
    inp = generate(cfg)
    L, B, d = cfg.L, cfg.B, cfg.d
    M, N, K = L * B, cfg.N, d

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    def f32(a):
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)

    X, W = bf16(inp["X"]), bf16(inp["W"])
    x, v, b, c0, dh = f32(inp["x"]), f32(inp["v"]), f32(inp["bias"]), f32(inp["c0"]), f32(inp["dh"])
    U = torch.empty(L, B, 1, 3, d, device=dev, dtype=torch.bfloat16)
    h = torch.empty(L, B, 1, d, device=dev)
    cT = torch.empty(B, 1, d, device=dev)
    ws = sru.alloc_workspace(L, B, d, False, device=dev)
    dU = torch.empty_like(U)
    dx = torch.empty(L, B, d, device=dev)
    dv = torch.empty(1, 2, d, device=dev)
    db = torch.empty(1, 2, d, device=dev)
    dc0 = torch.empty(B, 1, d, device=dev)
    dW = torch.empty(N, K, device=dev)
    stream = torch.cuda.current_stream(dev)
    reducer = None
    from parallelizable_recurrence_b200.dist import GradReducer
    if world > 1:
        reducer = GradReducer([dW, dv, db])  # one NCCL all-reduce of the parameter gradients

    fused = args.forward == "fused"
    names = (["forward_fused"] if fused else ["project", "forward"]) + ["backward", "project_dX", "project_dW"]

    def step(ev=None, bufs=None):
        """One training step; bufs = (X, x, dh, dx, dW, dv, db, dc0, reducer) or the default set.
        ev: CUDA events recorded between the phases (len(names) + 1)."""
        Xb, xb, dhb, dxb, dWb, dvb, dbb, dc0b, red = (bufs if bufs is not None
                                                      else (X, x, dh, dx, dW, dv, db, dc0, reducer))
        marks = iter(ev) if ev is not None else None

        def mark():
            if marks is not None:
                next(marks).record(stream)
        mark()
        if fused:  # Eq. (1) and Eqs. (2)-(5) in one kernel; U and the checkpoints stored for the backward
            sru.sru_forward_fused(Xb, W, xb, v, b, h, cT, ws, c0=c0, U=U)
            mark()
        else:
            sru.sru_project(Xb, W, U)
            mark()
            sru.sru_forward(U, xb, v, b, h, cT, c0=c0, workspace=ws)
            mark()
        sru.sru_backward(U, xb, v, b, dhb, ws, dU, dxb, dvb, dbb, dc0b, c0=c0)
        mark()
        sru.sru_project_backward(dU, Xb, W, dX=dxb, accumulate=True)
        mark()
        sru.sru_project_backward(dU, Xb, W, dW=dWb)
        mark()
        if red is not None:  # data-parallel gradient sum over ranks (batch sharding)
            red()

    for _ in range(args.warmup):
        step()
    st = sru.sru_sync_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    # ---- device-timed region
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    elapsed_ms = start.elapsed_time(stop)
    clocks = clk.summary()
    st = sru.sru_sync_status()
    if st != 0:
        raise RuntimeError(f"device status {st} in the timed region")
    phase_ms = {n: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps))
                for i, n in enumerate(names)}
    t = torch.tensor([elapsed_ms], device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    elapsed_ms = float(t.item())

    # ---- end to end: every step copies its inputs (X bf16, x and dh fp32) from
    # pinned host memory and reads its gradients (dx, dW, dv, db, dc0) back.  The
    # copies run on their own streams, double-buffered, so step k+1's inputs
    # travel while step k computes and step k's gradients travel back while
    # step k+1 computes (PCIe is full duplex).
    hX = torch.from_numpy(np.ascontiguousarray(inp["X"]).view(np.int16)).pin_memory()
    hx = torch.from_numpy(inp["x"]).pin_memory()
    hdh = torch.from_numpy(inp["dh"]).pin_memory()
    sets = []
    for i in range(2):
        Xi = X if i == 0 else torch.empty_like(X)
        xi = x if i == 0 else torch.empty_like(x)
        dhi = dh if i == 0 else torch.empty_like(dh)
        dxi = dx if i == 0 else torch.empty_like(dx)
        dWi = dW if i == 0 else torch.empty_like(dW)
        dvi = dv if i == 0 else torch.empty_like(dv)
        dbi = db if i == 0 else torch.empty_like(db)
        dc0i = dc0 if i == 0 else torch.empty_like(dc0)
        red = reducer if i == 0 or world == 1 else GradReducer([dWi, dvi, dbi])
        small = torch.empty(4 * d + B * d, device=dev)
        out_dW = torch.empty(N, K).pin_memory()
        out_dx = torch.empty(L, B, d).pin_memory()
        out_small = torch.empty(4 * d + B * d).pin_memory()
        sets.append(dict(bufs=(Xi, xi, dhi, dxi, dWi, dvi, dbi, dc0i, red), small=small, out_dW=out_dW,
                         out_dx=out_dx, out_small=out_small))
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in_ready", "computed", "out_done")}

    def e2e_run(nsteps, start_ev=None):
        if start_ev is not None:
            s_h2d.wait_event(start_ev)
        for k in range(nsteps):
            i = k % 2
            st_ = sets[i]
            Xi, xi, dhi, dxi, dWi, dvi, dbi, dc0i, _ = st_["bufs"]
            if k >= 2:
                s_h2d.wait_event(ev["computed"][i])  # step k-2 is done reading this input set
            with torch.cuda.stream(s_h2d):
                Xi.view(torch.int16).copy_(hX, non_blocking=True)
                xi.copy_(hx, non_blocking=True)
                dhi.copy_(hdh, non_blocking=True)
                ev["in_ready"][i].record(s_h2d)
            stream.wait_event(ev["in_ready"][i])
            if k >= 2:
                stream.wait_event(ev["out_done"][i])  # step k-2's gradients have left this set
            step(bufs=st_["bufs"])
            sm = st_["small"]
            sm[:2 * d].copy_(dvi.view(-1))
            sm[2 * d:4 * d].copy_(dbi.view(-1))
            sm[4 * d:].copy_(dc0i.view(-1))
            ev["computed"][i].record(stream)
            s_d2h.wait_event(ev["computed"][i])
            with torch.cuda.stream(s_d2h):
                st_["out_dW"].copy_(dWi, non_blocking=True)
                st_["out_dx"].copy_(dxi, non_blocking=True)
                st_["out_small"].copy_(sm, non_blocking=True)
                ev["out_done"][i].record(s_d2h)
        stream.wait_stream(s_h2d)
        stream.wait_stream(s_d2h)

    e2e_run(max(2, args.warmup))
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(args.steps, start_ev=e0)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    t = torch.tensor([e2e_ms], device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.barrier()
    e2e_ms = float(t.item())
    h2d = hX.numel() * 2 + hx.numel() * 4 + hdh.numel() * 4
    d2h = (sets[0]["out_dW"].numel() + sets[0]["out_dx"].numel() + sets[0]["out_small"].numel()) * 4
    st = sru.sru_sync_status()
    if st != 0:
        raise RuntimeError(f"device status {st} in the end-to-end region")

    workloads = None
    if rank == 0 and world == 1 and not args.skip_workloads:
        workloads = measure_workloads(dev, peaks)

    if rank == 0:
        tokens = cfg.tokens * world * args.steps
        value = tokens / (elapsed_ms / 1e3)
        gemm_flops = 2.0 * M * N * K
        traffic, traffic_src = load_traffic()
        traffic = traffic.get(WORKLOAD, {})
        tensor_phases = [n for n in ("forward_fused", "project", "project_dX", "project_dW") if n in phase_ms]
        gemm_ms = {n: phase_ms[n] for n in tensor_phases}
        dom = max(gemm_ms, key=gemm_ms.get)
        peak_kind, peak_tc = tensor_peak(peaks, clocks)
        ach_tc = gemm_flops / (gemm_ms[dom] / 1e3) / 1e12
        fwd_bytes = 14.0 * L * B * d
        bwd_bytes = 24.0 * L * B * d
        # the fused forward moves X, W, x, h and U (stored for the backward) instead of U twice
        fused_bytes = 2.0 * L * B * d + 6.0 * d * d + 14.0 * L * B * d
        ach_f = (fused_bytes if fused else fwd_bytes) / (phase_ms["forward_fused" if fused else "forward"] / 1e3) / 1e9
        ach_b = bwd_bytes / (phase_ms["backward"] / 1e3) / 1e9
        sm = clocks.get("sm_mhz")
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 GEMM + f32 recurrence",
            "data": "synthetic", "config": config,
            "roofline": {"bound": "tensor",
                         "kernel": ("sru_fused_fwd_kernel (forward_fused)" if dom == "forward_fused"
                                    else f"tc_gemm_pair_kernel ({dom})"), "achieved": ach_tc,
                         "peak": peak_tc, "unit": "TFLOP/s", "frac": ach_tc / peak_tc,
                         "traffic": traffic.get(dom), "traffic_unit": "bytes per launch (ncu dram read+write)",
                         "traffic_source": traffic_src,
                         "peak_source": f"{peaks['source']} bf16 {peak_kind} (chosen from this run's clocks: "
                                        f"median {sm} MHz, reasons {clocks.get('reasons')})",
                         "frac_of_burst": ach_tc / peaks["bf16_tflops"],
                         "frac_of_sustained": ach_tc / peaks["bf16_tflops_sustained"],
                         "frac_of_nominal_2250": ach_tc / NOMINAL_BF16_TFLOPS,
                         "ms_x_sm_mhz": gemm_ms[dom] * sm if sm else None,
                         "algorithmic_per_launch": f"2*M*N*K = {gemm_flops:.4g} flop"},
            "roofline_recurrence": {
                "bound": "hbm", "unit": "GB/s", "peak": peaks["hbm_gbs"],
                "forward": {"achieved": ach_f, "frac": ach_f / peaks["hbm_gbs"],
                            "bytes": fused_bytes if fused else fwd_bytes,
                            "kernel": "sru_fused_fwd_kernel (projection fused; the product bounds it)" if fused
                            else "sru_fwd_seq_kernel",
                            "ms": phase_ms["forward_fused" if fused else "forward"],
                            "traffic": traffic.get("forward_fused" if fused else "forward")},
                "backward": {"achieved": ach_b, "frac": ach_b / peaks["hbm_gbs"], "bytes": bwd_bytes,
                             "ms": phase_ms["backward"], "traffic": traffic.get("backward")},
                "traffic_source": traffic_src,
                "frac_of_nominal_8TBs": {"forward": ach_f / NOMINAL_HBM_GBS, "backward": ach_b / NOMINAL_HBM_GBS}},
            "phase_ms": phase_ms,
            "e2e": {"value": cfg.tokens * world * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            # per step: [sru_project, sru_forward | sru_forward_fused], the backward recurrence, the dv/db
            # reduction, dX, the zeroing of dW's split tail tiles, dW
            "gpu_launches": (6 if fused else 7) * args.steps,
            "forward_path": args.forward,
            "clocks": clocks,
        }
        if workloads is not None:
            line["workloads"] = workloads
        if world == 1:
            cpu_tps, desc, _, measured = cpu_baseline(cfg, budget_s=args.cpu_budget)
            line["cpu_baseline"] = {"value": cpu_tps, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                    "sample": desc, "extrapolated": True, "measured_s": measured, **host_info()}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


DECODE_METRIC = "SRU decode tokens/s (batch 1, one token through a stack of layers) and W-stream HBM GB/s on 1 B200"


def run_decode(args):
    """Token-by-token inference through a stack of unidirectional SRU layers
    (sru_decode_step: the per-token projection fused with Eqs. (2)-(5)).
    Every layer has its own W_cat, so a token streams layers * 6 d^2 bytes of
    weights, far more than L2: each step reads its W from HBM.  Each layer
    reads the same bf16 input row (the cast of one layer's h to the next
    layer's bf16 input is not part of the step being measured)."""
    import torch
    import torch.distributed as dist

    import parallelizable_recurrence_b200 as sru

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    sru.load_library()
    peaks = load_peaks()
    d, B, layers = 4096, 1, 8
    g = torch.Generator(device="cpu").manual_seed(1234 + rank)
    lim = (3.0 / d) ** 0.5
    Ws = [((torch.rand(3 * d, d, generator=g) * 2 - 1) * lim).to(dev, torch.bfloat16) for _ in range(layers)]
    vs = [(torch.rand(2, d, generator=g) - 0.5).to(dev) for _ in range(layers)]
    bs = [(torch.randn(2, d, generator=g) * 0.1).to(dev) for _ in range(layers)]
    cs = [torch.zeros(B, d, device=dev) for _ in range(layers)]
    hs = [torch.empty(B, d, device=dev) for _ in range(layers)]
    Xt = torch.randn(B, d, generator=g).to(dev, torch.bfloat16)
    xt = Xt.float()
    stream = torch.cuda.Stream(dev)

    def token():
        for l in range(layers):
            sru.sru_decode_step(Xt, Ws[l], xt, vs[l], bs[l], cs[l], hs[l], stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            token()
    torch.cuda.synchronize(dev)
    if sru.sru_sync_status() != 0:
        raise RuntimeError("device status after warm-up")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        token()
    graph.replay()
    torch.cuda.synchronize(dev)

    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(args.steps):
                graph.replay()
            stop.record(stream)
        torch.cuda.synchronize(dev)
    elapsed_ms = start.elapsed_time(stop)
    t = torch.tensor([elapsed_ms], device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    elapsed_ms = float(t.item())

    # end to end: per token, the input row goes up from pinned host memory and
    # the last layer's h comes back before the next token (autoregressive, so
    # nothing overlaps across tokens)
    hX = torch.from_numpy(np.ascontiguousarray(Xt.view(torch.int16).cpu().numpy())).pin_memory()
    hx = xt.cpu().pin_memory()
    hh = torch.empty(B, d).pin_memory()
    Xt16 = Xt.view(torch.int16)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            Xt16.copy_(hX, non_blocking=True)
            xt.copy_(hx, non_blocking=True)
            graph.replay()
            hh.copy_(hs[-1], non_blocking=True)
            stream.synchronize()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    del graph
    if sru.sru_sync_status() != 0:
        raise RuntimeError("device status in the timed region")

    if rank == 0:
        tok_s = world * args.steps / (elapsed_ms / 1e3)
        w_bytes = 6.0 * d * d * layers
        ach = w_bytes * args.steps / (elapsed_ms / 1e3) / 1e9
        line = {
            "metric": DECODE_METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 weights, f32 accumulate and state",
            "data": "synthetic",
            "config": {"workload": f"decode: {layers} unidirectional SRU layers d={d}, batch {B}, one token per "
                                   f"step, each layer's W_cat distinct ({w_bytes / 1e6:.0f} MB per token)",
                       "layers": layers, "d": d, "B": B, "graph": "one CUDA graph per token (8 launches)",
                       "l2": "weights per token 805 MB vs 126 MB L2; no flush"},
            "roofline": {"bound": "hbm", "kernel": "sru_decode_step_kernel<1>", "achieved": ach,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"], "traffic": None,
                         "algorithmic_per_launch": f"6*d*d = {6.0 * d * d:.4g} B of W (+ 5*d*4 B of state)"},
            "layer_step_us": elapsed_ms * 1e3 / (args.steps * layers),
            "e2e": {"value": world * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": B * d * 6, "d2h_bytes_per_step": B * d * 4},
            "gpu_launches": layers * args.steps,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_reference(args):
    """The oracle as it stands, on the host cores, same workload/metric; rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    cfg, config = workload_config()
    per_step = []
    desc = ""
    budget = args.ref_step_budget
    if budget is None:
        budget = min(2.0, 150.0 / max(1, args.warmup + args.steps))
    measured = []
    for k in range(args.warmup + args.steps):
        tps, desc, full, meas = cpu_baseline(cfg, budget_s=budget, seed=k)
        if k >= args.warmup:
            per_step.append(full)
            measured.append(meas)
    full_s = statistics.mean(per_step)
    value = cfg.tokens / full_s
    # ms_per_step is extrapolated from the measured sample (a full step of the
    # oracle would take hours); the seconds actually measured are given beside it
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": full_s * 1e3, "extrapolated": True,
            "measured_sample_s_per_step": statistics.mean(measured), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc,
                             "extrapolated": True, "measured_s": statistics.mean(measured), **host_info()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def run_only(args):
    """One layer of the per-workload block alone (e.g. under ncu -k <kernel>)."""
    import torch
    import parallelizable_recurrence_b200 as sru
    torch.cuda.set_device(0)
    sru.load_library()
    out = measure_workloads(torch.device("cuda", 0), load_peaks(), only=args.only)
    print(json.dumps({"only": args.only, **out}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["train", "decode"], default="train",
                    help="train: the layer training step (the headline); decode: batch-1 token steps")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--forward", choices=["fused", "separate"], default="fused",
                    help="training step's forward: sru_forward_fused (projection and recurrence in one kernel) or "
                         "sru_project then sru_forward")
    ap.add_argument("--only", choices=sorted(WORKLOAD_LAYERS), default=None,
                    help="run only this layer of the per-workload block and print it (for profiling one kernel)")
    ap.add_argument("--skip-workloads", action="store_true",
                    help="leave out the per-workload block (the headline step only)")
    ap.add_argument("--ref-step-budget", type=float, default=None,
                    help="seconds of oracle work per reference step (default: 2 s, less so that the whole "
                         "--impl reference run stays near 150 s)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.only is not None:
        run_only(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.workload == "decode":
        run_decode(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
