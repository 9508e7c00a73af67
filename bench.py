"""Benchmark of the deformable sampling-aggregation forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload NAME] [--pass forward|backward]

One step is one dcn_forward (or msda_forward) call over one full batch of the
workload; the default workload is DCNv4 fp16, N=64, 56x56, C=64, G=4, 3x3.
`--pass backward` times dcn_backward (msda_backward) instead: one call = the
zero fill of the float32 accumulator, the gradient kernel and the rounding.
Prints ONE JSON line on stdout (rank 0); diagnostics go to stderr.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and a device synchronisation on both sides, timed with CUDA events on the
launch stream.  The steps rotate over enough independent input/output sets
that their total exceeds three L2 caches, so every step reads from HBM.
Multi-GPU (torchrun): each rank runs its own batch (weak scaling, no data
collective); the time is the maximum over ranks and `value` counts the taps
of all ranks.

`--impl reference` times the float64 CPU oracle (the reference arm) on rank 0
over a bounded sample of the same workload per step.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gen  # noqa: E402

METRIC = ("sampled taps/s & achieved HBM GB/s vs peak "
          "(DCNv4 fp16 fwd, 64×56²×64, G=4)")
# Random 32-byte gathers that hit in L1 move at most this many bytes per SM
# clock on B200 (measured with a random ld.global.nc.v8 probe, L1-resident
# footprint; the rate falls to about 30 B/clk when the footprint spills to L2).
L1_GATHER_BYTES_PER_CLK = 58.0
FALLBACK_HBM_GBS = 6650.0
# Shared memory delivers 32 banks x 4 bytes per SM clock to conflict-free reads.
SMEM_BYTES_PER_CLK = 128.0
# Float32 reductions into random 32-byte sectors (two lanes per sector,
# red.global.add.v4.f32) reach about this many bytes per SM clock on B200
# (measured with a reduction probe: 120 G sectors/s over 148 SMs at 1965 MHz).
REDUCTION_BYTES_PER_CLK = 13.2
# Random 128-byte rows (four lanes of 32 bytes each, ld.global.nc) gathered
# from a 40 MB L2-resident float32 tensor reach about this many bytes per SM
# clock on B200 (measured: 141 G rows/s over 148 SMs at 1965 MHz; TMA
# tile::gather4 loads of the same rows reached at most 46 G rows/s).
ROW_GATHER_BYTES_PER_CLK = 62.0

# DRAM traffic of the timed kernel from one ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum per launch, headline workload), with the hash of the
# files the headline launch is built from; reported as null once they change.
NCU_TRAFFIC = {
    "source_sha256": "703c22acb9f78b6ae3888b2bc27e956b3a9d546e764e74ebdab5b89050d03905",
    "bytes_per_launch": 69778432 + 3547904,   # DRAM read + write, one headline launch
}

# What the headline dcn_forward launch is built from: its device code and the
# host code that validates, chooses the launch shape and dispatches it.
FORWARD_SOURCES = [
    "deformable_attention_sampling_b200/csrc/common.cuh",
    "deformable_attention_sampling_b200/csrc/dcn_fwd.cuh",
    "deformable_attention_sampling_b200/csrc/dcn_band.cuh",
    "deformable_attention_sampling_b200/csrc/abi_common.cuh",
    "deformable_attention_sampling_b200/csrc/abi_common.cu",
    "deformable_attention_sampling_b200/csrc/abi_dcn_fwd.cu",
]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def kernel_source_hash():
    h = hashlib.sha256()
    for p in FORWARD_SOURCES:
        path = os.path.join(ROOT, p)
        if os.path.exists(path):
            h.update(p.encode())
            with open(path, "rb") as f:
                h.update(f.read())
    return h.hexdigest()


def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock, max clock and clock-event reasons with NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index):
        self.samples = []
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            props = torch.cuda.get_device_properties(device_index)
            handle = None
            for lookup in (
                    lambda: pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid)),
                    lambda: pynvml.nvmlDeviceGetHandleByPciBusId(
                        f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:"
                        f"{props.pci_device_id:02X}.0"),
                    lambda: pynvml.nvmlDeviceGetHandleByIndex(device_index)):
                try:
                    handle = lookup()
                    break
                except Exception:
                    continue
            if handle is None:
                raise RuntimeError("no NVML handle for the CUDA device")
            self.handle = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:   # no NVML: report the clocks as unavailable
            self.nvml = None
            self.error = str(e)

    def _sample(self):
        n = self.nvml
        sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
        try:
            reasons = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
        except AttributeError:
            reasons = n.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
        self.samples.append((sm, reasons))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception as e:
                self.error = str(e)
                return
            time.sleep(0.002)

    def start(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            try:
                self._sample()      # at least one sample right at the end
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "error": self.error}
        mask = 0
        for _, r in self.samples:
            mask |= int(r)
        reasons = [name for bit, name in self.REASONS.items() if mask & bit]
        return {"sm_mhz": statistics.median(s for s, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


def on_chip_roofline(w, ms_per_launch, sampler, device, band=False):
    """The SM-side bound: every tap reads four corner vectors of D channels
    (the kernels load all four, out-of-map ones from a clamped address with
    zero weight).  The gather kernel reads them through L1: peak = the
    measured L1 rate of random 32-byte gathers x SMs x the median SM clock
    sampled during the timed region.  The band kernel reads them from shared
    memory with conflict-free 16-byte lanes: peak = 128 bytes per SM clock
    (32 banks x 4 bytes) x SMs x the same clock."""
    es = gen.DTYPES[w.dtype].itemsize
    gathered = w.taps() * 4 * w.D * es
    achieved = gathered / (ms_per_launch * 1e-3) / 1e9
    clocks = sampler.summary()
    mhz = clocks["sm_mhz"] or clocks["sm_max_mhz"] or 1965
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    rate = SMEM_BYTES_PER_CLK if band else L1_GATHER_BYTES_PER_CLK
    peak = rate * sms * mhz * 1e6 / 1e9
    basis = ("128 B/clk/SM shared-memory bandwidth (32 banks x 4 B)" if band else
             f"{L1_GATHER_BYTES_PER_CLK:g} B/clk/SM measured random 32 B gathers")
    return {"bound": "smem" if band else "l1_gather", "achieved": achieved, "peak": peak,
            "unit": "GB/s", "frac": achieved / peak, "gathered_bytes_per_launch": gathered,
            "peak_basis": f"{basis} x {sms} SMs x {mhz} MHz"}


def reduction_roofline(w, ms_per_call, sampler, device):
    """The bound of a DCN backward call: its grad_x scatter adds four corner
    vectors of D float32 channels per tap, as whole 32-byte sectors at random
    positions (corners outside the map are skipped, so this slightly
    overcounts), against the measured random-sector reduction rate x SMs x
    the median sampled SM clock.  (MSDA's corners are whole 128-byte rows, a
    pattern this rate does not describe.)"""
    scattered = w.taps() * 4 * w.D * 4
    achieved = scattered / (ms_per_call * 1e-3) / 1e9
    clocks = sampler.summary()
    mhz = clocks["sm_mhz"] or clocks["sm_max_mhz"] or 1965
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    peak = REDUCTION_BYTES_PER_CLK * sms * mhz * 1e6 / 1e9
    return {"bound": "l2_reduction", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "reduced_bytes_per_call": scattered,
            "peak_basis": f"{REDUCTION_BYTES_PER_CLK:g} B/clk/SM measured random-sector float32 "
                          f"reductions x {sms} SMs x {mhz} MHz"}


def row_gather_roofline(w, ms_per_launch, sampler, device):
    """The SM-side bound of an MSDA forward: every tap reads four corner rows
    of D channels (a (pixel, head) row of the value tensor, out-of-map ones
    from a clamped row with zero weight), at data-dependent positions in a
    value tensor that stays in L2, against the measured rate of random
    128-byte row gathers from L2 x SMs x the median sampled SM clock."""
    es = gen.DTYPES[w.dtype].itemsize
    gathered = w.taps() * 4 * w.D * es
    achieved = gathered / (ms_per_launch * 1e-3) / 1e9
    clocks = sampler.summary()
    mhz = clocks["sm_mhz"] or clocks["sm_max_mhz"] or 1965
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    peak = ROW_GATHER_BYTES_PER_CLK * sms * mhz * 1e6 / 1e9
    return {"bound": "l2_row_gather", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "gathered_bytes_per_launch": gathered,
            "peak_basis": f"{ROW_GATHER_BYTES_PER_CLK:g} B/clk/SM measured random 128-byte row "
                          f"gathers from L2 x {sms} SMs x {mhz} MHz"}


def fma_roofline(w, ms_per_launch, sampler, device):
    """The arithmetic side of the ContMix core: one float32 FMA per (location,
    tap, channel), against the SMs' float32 FMA rate (128 lanes per SM per
    clock) at the median SM clock sampled during the timed region."""
    fmas = w.taps() * w.D
    achieved = 2 * fmas / (ms_per_launch * 1e-3) / 1e12
    clocks = sampler.summary()
    mhz = clocks["sm_mhz"] or clocks["sm_max_mhz"] or 1965
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    peak = 2 * 128 * sms * mhz * 1e6 / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "fma_per_launch": fmas,
            "peak_basis": f"128 FP32 FMA lanes x {sms} SMs x {mhz} MHz"}


# ------------------------------------------------------------------ runners

class DcnRunner:
    algo = 0     # DCN_ALGO_AUTO; set from --algo

    def __init__(self, w, seed, device):
        import deformable_attention_sampling_b200 as dcnb
        self.dcnb = dcnb
        self.w = w
        self.host = gen.dcn_inputs(w, seed=seed)
        self.device = device
        self.code = gen.DTYPE_CODES[w.dtype]
        self.lib = dcnb.library()

    def alloc_set(self):
        d = {k: v.to(self.device) for k, v in self.host.items()}
        d["out"] = torch.empty((self.w.N, self.w.Ho, self.w.Wo, self.w.C),
                               dtype=self.host["x"].dtype, device=self.device)
        return d

    def launcher(self, s, stream):
        """A closure issuing one step on set s with pre-resolved arguments."""
        w, lib = self.w, self.lib
        args = (s["x"].data_ptr(), s["offset"].data_ptr(), s["mask"].data_ptr(),
                s["out"].data_ptr(), w.N, w.H, w.W, w.C, w.G, w.kh, w.kw, w.stride, w.pad,
                w.dil, w.softmax_flag, self.code, self.algo, stream)

        def go():
            st = lib.dcn_forward_algo(*args)
            if st != 0:
                raise self.dcnb.DcnError(st, "dcn_forward_algo")
        return go

    def inputs_of(self, s):
        return [(s["x"], self.host["x"]), (s["offset"], self.host["offset"]),
                (s["mask"], self.host["mask"])]

    def outputs_of(self, s):
        return [s["out"]]

    kernel = "dcn_fwd_kernel"

    def bytes_per_step(self):
        return self.w.compulsory_bytes()


class MsdaRunner:
    def __init__(self, w, seed, device):
        import deformable_attention_sampling_b200 as dcnb
        self.dcnb = dcnb
        self.w = w
        self.host = {k: v for k, v in gen.msda_inputs(w, seed=seed).items() if k != "logits"}
        self.device = device
        self.code = gen.DTYPE_CODES[w.dtype]
        self.lib = dcnb.library()

    def alloc_set(self):
        d = {k: v.to(self.device) for k, v in self.host.items()}
        d["out"] = torch.empty((self.w.N, self.w.queries, self.w.M * self.w.D),
                               dtype=self.host["value"].dtype, device=self.device)
        return d

    def launcher(self, s, stream):
        w, lib = self.w, self.lib
        args = (s["value"].data_ptr(), s["spatial_shapes"].data_ptr(),
                s["level_start"].data_ptr(), s["loc"].data_ptr(), s["attn"].data_ptr(),
                s["out"].data_ptr(), w.N, w.queries, w.M, w.D, w.L, w.K, self.code, stream)

        def go():
            st = lib.msda_forward(*args)
            if st != 0:
                raise self.dcnb.DcnError(st, "msda_forward")
        return go

    def inputs_of(self, s):
        return [(s[k], self.host[k]) for k in ("value", "spatial_shapes", "level_start", "loc",
                                               "attn")]

    def outputs_of(self, s):
        return [s["out"]]

    kernel = "msda_fwd_kernel"

    def bytes_per_step(self):
        return self.w.compulsory_bytes()


class DcnBwdRunner(DcnRunner):
    """One step = one dcn_backward call: zero fill of the float32 grad_x
    accumulator, the gradient kernel, rounding into grad_x (16-bit data)."""
    kernel = "dcn_bwd_kernel (+ zero fill, rounding)"

    def __init__(self, w, seed, device):
        super().__init__(w, seed, device)
        self.host["grad_out"] = gen.grad_out((w.N, w.Ho, w.Wo, w.C), w.dtype, seed)
        self.ws_bytes = self.dcnb.dcn_backward_workspace_size(w.N, w.H, w.W, w.C, self.code)

    def alloc_set(self):
        d = {k: v.to(self.device) for k, v in self.host.items()}
        d["grad_x"] = torch.empty_like(d["x"])
        d["grad_offset"] = torch.empty_like(d["offset"])
        d["grad_mask"] = torch.empty_like(d["mask"])
        d["ws"] = (torch.empty(self.ws_bytes // 4, dtype=torch.float32, device=self.device)
                   if self.ws_bytes > 0 else None)
        return d

    def launcher(self, s, stream):
        w, lib = self.w, self.lib
        ws = s["ws"].data_ptr() if s["ws"] is not None else None
        args = (s["x"].data_ptr(), s["offset"].data_ptr(), s["mask"].data_ptr(),
                s["grad_out"].data_ptr(), s["grad_x"].data_ptr(), s["grad_offset"].data_ptr(),
                s["grad_mask"].data_ptr(), ws, self.ws_bytes, w.N, w.H, w.W, w.C, w.G, w.kh,
                w.kw, w.stride, w.pad, w.dil, w.softmax_flag, self.code, stream)

        def go():
            st = lib.dcn_backward(*args)
            if st != 0:
                raise self.dcnb.DcnError(st, "dcn_backward")
        return go

    def inputs_of(self, s):
        return super().inputs_of(s) + [(s["grad_out"], self.host["grad_out"])]

    def outputs_of(self, s):
        return [s["grad_x"], s["grad_offset"], s["grad_mask"]]

    def bytes_per_step(self):
        return self.w.backward_bytes()


class MsdaBwdRunner(MsdaRunner):
    """One step = one msda_backward call (zero fill, gradient kernel, and the
    rounding pass for 16-bit data)."""
    kernel = "msda_bwd_kernel (+ zero fill, rounding)"

    def __init__(self, w, seed, device):
        super().__init__(w, seed, device)
        self.host["grad_out"] = gen.grad_out((w.N, w.queries, w.M * w.D), w.dtype, seed)
        self.ws_bytes = self.dcnb.msda_backward_workspace_size(w.N, w.S, w.M, w.D, self.code)

    def alloc_set(self):
        d = {k: v.to(self.device) for k, v in self.host.items()}
        d["grad_value"] = torch.empty_like(d["value"])
        d["grad_loc"] = torch.empty_like(d["loc"])
        d["grad_attn"] = torch.empty_like(d["attn"])
        d["ws"] = (torch.empty(self.ws_bytes // 4, dtype=torch.float32, device=self.device)
                   if self.ws_bytes > 0 else None)
        return d

    def launcher(self, s, stream):
        w, lib = self.w, self.lib
        ws = s["ws"].data_ptr() if s["ws"] is not None else None
        args = (s["value"].data_ptr(), s["spatial_shapes"].data_ptr(),
                s["level_start"].data_ptr(), s["loc"].data_ptr(), s["attn"].data_ptr(),
                s["grad_out"].data_ptr(), s["grad_value"].data_ptr(), s["grad_loc"].data_ptr(),
                s["grad_attn"].data_ptr(), ws, self.ws_bytes, w.N, w.S, w.queries, w.M, w.D,
                w.L, w.K, self.code, stream)

        def go():
            st = lib.msda_backward(*args)
            if st != 0:
                raise self.dcnb.DcnError(st, "msda_backward")
        return go

    def inputs_of(self, s):
        return super().inputs_of(s) + [(s["grad_out"], self.host["grad_out"])]

    def outputs_of(self, s):
        return [s["grad_value"], s["grad_loc"], s["grad_attn"]]

    def bytes_per_step(self):
        return self.w.backward_bytes()


class DynRunner:
    """One step = one dynconv_forward_algo call (the ContMix core)."""
    kernel = "dynconv_fwd_kernel"
    algo = 0     # DCN_ALGO_AUTO; set from --algo

    def __init__(self, w, seed, device):
        import deformable_attention_sampling_b200 as dcnb
        self.dcnb = dcnb
        self.w = w
        self.host = gen.dynconv_inputs(w, seed=seed)
        self.device = device
        self.code = gen.DTYPE_CODES[w.dtype]
        self.lib = dcnb.library()

    def alloc_set(self):
        d = {k: v.to(self.device) for k, v in self.host.items()}
        d["out"] = torch.empty_like(d["x"])
        return d

    def launcher(self, s, stream):
        w, lib = self.w, self.lib
        args = (s["x"].data_ptr(), s["weights"].data_ptr(), s["out"].data_ptr(), w.N, w.H, w.W,
                w.C, w.G, w.K, w.softmax_flag, self.code, self.algo, stream)

        def go():
            st = lib.dynconv_forward_algo(*args)
            if st != 0:
                raise self.dcnb.DcnError(st, "dynconv_forward_algo")
        return go

    def inputs_of(self, s):
        return [(s["x"], self.host["x"]), (s["weights"], self.host["weights"])]

    def outputs_of(self, s):
        return [s["out"]]

    def bytes_per_step(self):
        return self.w.compulsory_bytes()


class MsdaPointsRunner:
    """One step = one msda_forward_points call (locations formed in-kernel
    from box / point references and valid ratios)."""
    kernel = "msda_fwd_kernel (reference-point variant)"

    def __init__(self, w, seed, device):
        import deformable_attention_sampling_b200 as dcnb
        self.dcnb = dcnb
        self.w = w
        self.host = {k: v for k, v in gen.msda_ref_inputs(w, seed=seed).items() if k != "mask"}
        self.device = device
        self.code = gen.DTYPE_CODES[w.dtype]
        self.lib = dcnb.library()

    def alloc_set(self):
        d = {k: v.to(self.device) for k, v in self.host.items()}
        d["out"] = torch.empty((self.w.N, self.w.queries, self.w.M * self.w.D),
                               dtype=self.host["value"].dtype, device=self.device)
        return d

    def launcher(self, s, stream):
        w, lib = self.w, self.lib
        args = (s["value"].data_ptr(), s["spatial_shapes"].data_ptr(),
                s["level_start"].data_ptr(), s["reference"].data_ptr(), w.ref_dim,
                s["valid_ratios"].data_ptr(), s["offsets"].data_ptr(), s["attn"].data_ptr(),
                s["out"].data_ptr(), w.N, w.queries, w.M, w.D, w.L, w.K, self.code, stream)

        def go():
            st = lib.msda_forward_points(*args)
            if st != 0:
                raise self.dcnb.DcnError(st, "msda_forward_points")
        return go

    def inputs_of(self, s):
        return [(s[k], self.host[k]) for k in ("value", "spatial_shapes", "level_start",
                                               "reference", "valid_ratios", "offsets", "attn")]

    def outputs_of(self, s):
        return [s["out"]]

    def bytes_per_step(self):
        return self.w.compulsory_bytes()


class FusedRunner:
    """One step = one dcnv4_fused_forward call (merged offset / mask linear on
    the tensor cores feeding the sampler; offsets never leave the SM)."""
    kernel = "dcn_band_fused_kernel (tcgen05 front end) where it applies, else dcn_fwd_kernel"

    def __init__(self, w, seed, device):
        import deformable_attention_sampling_b200 as dcnb
        self.dcnb = dcnb
        self.w = w
        self.host = gen.front_end_inputs(w, seed=seed)
        self.device = device
        self.code = gen.DTYPE_CODES[w.dtype]
        self.lib = dcnb.library()

    def alloc_set(self):
        d = {k: v.to(self.device) for k, v in self.host.items()}
        d["out"] = torch.empty_like(d["x"])
        return d

    def launcher(self, s, stream):
        w, lib = self.w, self.lib
        args = (s["x"].data_ptr(), s["w_om"].data_ptr(), s["b_om"].data_ptr(),
                s["out"].data_ptr(), w.N, w.H, w.W, w.C, w.G, w.kh, w.kw, w.pad, w.dil,
                self.code, stream)

        def go():
            st = lib.dcnv4_fused_forward(*args)
            if st != 0:
                raise self.dcnb.DcnError(st, "dcnv4_fused_forward")
        return go

    def inputs_of(self, s):
        return [(s[k], self.host[k]) for k in ("x", "w_om", "b_om")]

    def outputs_of(self, s):
        return [s["out"]]

    def bytes_per_step(self):
        return self.w.compulsory_bytes()


def make_runner(w, seed, device, backward=False):
    if isinstance(w, gen.FusedWorkload):
        if backward:
            raise SystemExit("--pass backward is not offered for the fused front end")
        return FusedRunner(w, seed, device)
    if isinstance(w, gen.MsdaWorkload) and w.ref_dim:
        if backward:
            raise SystemExit("--pass backward is not offered for the reference-point variants")
        return MsdaPointsRunner(w, seed, device)
    if isinstance(w, gen.DynWorkload):
        if backward:
            raise SystemExit("--pass backward is not offered for the ContMix workloads")
        return DynRunner(w, seed, device)
    dcn = isinstance(w, gen.DcnWorkload)
    if backward:
        return (DcnBwdRunner if dcn else MsdaBwdRunner)(w, seed, device)
    return (DcnRunner if dcn else MsdaRunner)(w, seed, device)


# ------------------------------------------------------------------ CPU oracle

def oracle_step(w, seed, backward=False):
    """Run the float64 oracle once on workload w; returns (seconds, taps)."""
    import oracle
    if backward and isinstance(w, gen.DcnWorkload):
        inp = gen.dcn_inputs(w, seed=seed)
        go = gen.grad_out((w.N, w.Ho, w.Wo, w.C), w.dtype, seed)
        t = time.perf_counter()
        oracle.dcn_backward_ref(inp["x"], inp["offset"], inp["mask"], go, w.kh, w.kw, w.stride,
                                w.pad, w.dil, w.softmax_flag)
    elif isinstance(w, gen.MsdaWorkload) and w.ref_dim:
        inp = gen.msda_ref_inputs(w, seed=seed)
        t = time.perf_counter()
        oracle.msda_points_ref(inp["value"], inp["spatial_shapes"], inp["level_start"],
                               inp["reference"], inp["offsets"], inp["attn"], inp["valid_ratios"])
    elif backward:
        inp = gen.msda_inputs(w, seed=seed)
        go = gen.grad_out((w.N, w.queries, w.M * w.D), w.dtype, seed)
        t = time.perf_counter()
        oracle.msda_backward_ref(inp["value"], inp["spatial_shapes"], inp["level_start"],
                                 inp["loc"], inp["attn"], go)
    elif isinstance(w, gen.FusedWorkload):
        inp = gen.front_end_inputs(w, seed=seed)
        t = time.perf_counter()
        oracle.dcnv4_front_end_ref(inp["x"], inp["w_om"], inp["b_om"], w.kh, w.kw, w.pad, w.dil,
                                   w.G)
    elif isinstance(w, gen.DynWorkload):
        inp = gen.dynconv_inputs(w, seed=seed)
        t = time.perf_counter()
        oracle.dynconv_forward_ref(inp["x"], inp["weights"], w.K, w.softmax_flag)
    elif isinstance(w, gen.DcnWorkload):
        inp = gen.dcn_inputs(w, seed=seed)
        t = time.perf_counter()
        oracle.dcn_forward_ref(inp["x"], inp["offset"], inp["mask"], w.kh, w.kw, w.stride,
                               w.pad, w.dil, w.softmax_flag)
    else:
        inp = gen.msda_inputs(w, seed=seed)
        t = time.perf_counter()
        oracle.msda_forward_ref(inp["value"], inp["spatial_shapes"], inp["level_start"],
                                inp["loc"], inp["attn"])
    return time.perf_counter() - t, w.taps()


def sample_of(w, n_images):
    """A bounded sample of workload w with the same per-tap work: fewer batch
    items (DCN) or fewer queries (MSDA)."""
    if isinstance(w, (gen.DcnWorkload, gen.DynWorkload, gen.FusedWorkload)):
        return gen.scaled(w, N=max(1, min(w.N, n_images)))
    return gen.scaled(w, N=1, Lq=max(1, min(w.queries, n_images * 64)))


def _oracle_worker(task):
    """One host process of the all-core leg: runs the oracle on its tasks
    (each a bounded sample with its own seed) and returns its busy time and
    taps.  Top-level so that a spawned process can import it."""
    w, seeds, backward = task
    busy, taps = 0.0, 0
    for seed in seeds:
        dt, t = oracle_step(w, seed=seed, backward=backward)
        busy += dt
        taps += t
    return busy, taps


def cpu_baseline(w, budget_s=10.0, backward=False, pool=None, cores=1):
    """The oracle as it stands on a bounded sample of the workload.

    Single-threaded: repeated until about budget_s / 2 seconds of CPU work.
    All cores: `pool` (spawned processes, one per host core) runs the same
    oracle on the same sample size, each process over its own seeds, about
    budget_s / 2 seconds per process; the rate is all taps over the busiest
    process's oracle time (input generation is outside the timed calls)."""
    s = sample_of(w, 8)
    total_t, total_taps, reps = 0.0, 0, 0
    while total_t < budget_s / 2 or reps == 0:
        dt, taps = oracle_step(s, seed=reps, backward=backward)
        total_t += dt
        total_taps += taps
        reps += 1
    single = total_taps / total_t
    what = (f"oracle on {s.name} with N={s.N}" +
            (f", Lq={s.queries}" if isinstance(s, gen.MsdaWorkload) else "") +
            f" ({s.taps()} taps each), float64" + (", backward" if backward else ""))
    result = {"value": single, "unit": "taps/s", "cores": 1, "kind": "oracle",
              "sample": f"{reps} x {what}, single thread", "host_cpus": os.cpu_count(),
              "single_thread_value": single}
    if pool is not None and cores > 1:
        per = max(1, int(round(budget_s / 2 / (total_t / reps))))
        tasks = [(s, [10_000 + c * per + i for i in range(per)], backward)
                 for c in range(cores)]
        parts = pool.map(_oracle_worker, tasks)
        busiest = max(b for b, _ in parts)
        taps_all = sum(t for _, t in parts)
        result.update({
            "value": taps_all / busiest, "cores": cores,
            "sample": (f"{cores} processes x {per} x {what}, one process per host core "
                       f"(rate = all taps / busiest process's oracle time); single thread: "
                       f"{reps} x the same sample"),
            "all_core_value": taps_all / busiest})
    return result


def start_oracle_pool(cores):
    """Host processes for the all-core oracle leg, started with `spawn` (a
    process forked after CUDA is initialised can hang)."""
    import multiprocessing as mp
    if cores <= 1:
        return None
    return mp.get_context("spawn").Pool(cores)


# ------------------------------------------------------------------ main arms

def setup_distributed():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(f"cuda:{local}"))
    return world, rank, local


def max_over_ranks(x, world, device):
    from deformable_attention_sampling_b200.sharding import max_over_ranks as reduce_max
    return reduce_max(x, device) if world > 1 else x


def barrier(world, device):
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[device.index])
    torch.cuda.synchronize(device)


def run_b200(args):
    # the all-core oracle leg's processes start before CUDA is initialised
    pool = None
    if int(os.environ.get("WORLD_SIZE", "1")) == 1:
        pool = start_oracle_pool(os.cpu_count() or 1)
    world, rank, local = setup_distributed()
    device = torch.device(f"cuda:{local}")
    torch.cuda.set_device(device)
    w = gen.WORKLOADS[args.workload]
    import deformable_attention_sampling_b200 as dcnb
    from deformable_attention_sampling_b200 import build as dcn_build
    if not os.path.exists(dcn_build.LIB):
        raise RuntimeError("libdcn_b200.so is not built (python -m "
                           "deformable_attention_sampling_b200.build)")

    backward = args.pass_ == "backward"
    runner = make_runner(w, seed=1000 + rank, device=device, backward=backward)
    band = False
    dyn_algos = ("auto", "simt", "tensor")
    if isinstance(runner, DynRunner) != (args.algo in dyn_algos[1:]) and args.algo != "auto":
        raise ValueError(f"--algo {args.algo} does not apply to workload {w.name}")
    if isinstance(runner, DynRunner):
        runner.algo = dcnb.DYNCONV_ALGO_CODES[args.algo]
        # which kernel the timed calls run: the tensor-core one where it applies
        tensor = False
        if args.algo != "simt":
            probe = runner.alloc_set()
            tensor = dcnb.library().dynconv_forward_algo(
                probe["x"].data_ptr(), probe["weights"].data_ptr(), probe["out"].data_ptr(),
                w.N, w.H, w.W, w.C, w.G, w.K, w.softmax_flag, runner.code,
                dcnb.DCN_ALGO_TENSOR, int(torch.cuda.current_stream(device).cuda_stream)) == 0
            torch.cuda.synchronize(device)
            del probe
        runner.kernel = ("dynconv_mma_kernel (mma.sync m16n8k16)" if tensor
                         else "dynconv_fwd_kernel")
    elif isinstance(runner, DcnRunner) and not backward:
        runner.algo = dcnb.ALGO_CODES[args.algo]
        # which kernel the timed calls run: the band kernel where it applies
        if args.algo != "gather":
            probe = runner.alloc_set()
            band = dcnb.library().dcn_forward_algo(
                probe["x"].data_ptr(), probe["offset"].data_ptr(), probe["mask"].data_ptr(),
                probe["out"].data_ptr(), w.N, w.H, w.W, w.C, w.G, w.kh, w.kw, w.stride, w.pad,
                w.dil, w.softmax_flag, runner.code, dcnb.DCN_ALGO_BAND,
                int(torch.cuda.current_stream(device).cuda_stream)) == 0
            torch.cuda.synchronize(device)
            del probe
        runner.kernel = "dcn_band_kernel" if band else "dcn_fwd_kernel"
    elif isinstance(runner, FusedRunner):
        probe = runner.alloc_set()
        fused_band = dcnb.library().dcnv4_fused_forward_algo(
            probe["x"].data_ptr(), probe["w_om"].data_ptr(), probe["b_om"].data_ptr(),
            probe["out"].data_ptr(), w.N, w.H, w.W, w.C, w.G, w.kh, w.kw, w.pad, w.dil,
            runner.code, dcnb.DCN_ALGO_BAND,
            int(torch.cuda.current_stream(device).cuda_stream)) == 0
        torch.cuda.synchronize(device)
        del probe
        runner.kernel = ("dcn_band_fused_kernel (tcgen05 front end)" if fused_band
                         else "dcn_fwd_kernel (fused front end, mma.sync)")
    bytes_per_step = runner.bytes_per_step()
    l2_bytes = torch.cuda.get_device_properties(device).L2_cache_size
    n_sets = max(2, int(np.ceil(3 * l2_bytes / bytes_per_step)))
    sets = [runner.alloc_set() for _ in range(n_sets)]
    stream = torch.cuda.current_stream(device)
    handle = int(stream.cuda_stream)
    launch = [runner.launcher(s, handle) for s in sets]
    log(f"[rank {rank}] workload {w.name}: {w.taps()} taps, {bytes_per_step / 1e6:.2f} MB "
        f"compulsory per step, {n_sets} rotating sets")

    for i in range(args.warmup):
        launch[i % n_sets]()
    barrier(world, device)

    sampler = ClockSampler(local)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    launches_before = dcnb.dcn_launch_count()
    sampler.start()
    start.record(stream)
    for i in range(args.steps):
        launch[i % n_sets]()
    end.record(stream)
    end.synchronize()
    sampler.stop()
    launches = dcnb.dcn_launch_count() - launches_before
    barrier(world, device)
    ms_local = start.elapsed_time(end)
    ms = max_over_ranks(ms_local, world, device)
    ms_per_step = ms / args.steps

    # end to end through the public call with host buffers: H2D of the step's
    # inputs from pinned memory, the call, D2H of the output, every step
    e2e_steps = min(args.steps, 200)
    pinned_out = [(torch.empty(o.shape, dtype=o.dtype).pin_memory(), o)
                  for o in runner.outputs_of(sets[0])]
    pinned_in = [(dev, host.pin_memory()) for dev, host in runner.inputs_of(sets[0])]
    h2d = sum(h.numel() * h.element_size() for _, h in pinned_in)
    d2h = sum(h.numel() * h.element_size() for h, _ in pinned_out)
    for _ in range(2):
        for dev, host in pinned_in:
            dev.copy_(host, non_blocking=True)
        launch[0]()
        for host, dev in pinned_out:
            host.copy_(dev, non_blocking=True)
    barrier(world, device)
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(e2e_steps):
        for dev, host in pinned_in:
            dev.copy_(host, non_blocking=True)
        launch[0]()
        for host, dev in pinned_out:
            host.copy_(dev, non_blocking=True)
    e_end.record(stream)
    e_end.synchronize()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), world, device) / e2e_steps
    barrier(world, device)

    taps_total = w.taps() * world
    value = taps_total / (ms_per_step * 1e-3)
    peak, peak_src = measured_hbm_peak()
    achieved = bytes_per_step / (ms_local / args.steps * 1e-3) / 1e9
    traffic = None
    if (NCU_TRAFFIC["source_sha256"] == kernel_source_hash()
            and w.name == gen.HEADLINE and not backward):
        traffic = NCU_TRAFFIC["bytes_per_launch"]

    result = None
    if rank == 0:
        kernel = runner.kernel
        config = {"workload": w.name, "global_batch": w.N * world,
                  "per_gpu_batch": w.N, "dtype_storage": w.dtype, "accumulate": "f32",
                  "l2": f"{n_sets} rotating input/output sets ({n_sets * bytes_per_step / 1e6:.0f} MB"
                        f" > 3 x L2 {l2_bytes / 1e6:.0f} MB)",
                  "parallelism": f"dp{world}" if world > 1 else "single GPU"}
        if isinstance(w, gen.FusedWorkload):
            config.update({"H": w.H, "W": w.W, "C": w.C, "G": w.G, "kernel": f"{w.kh}x{w.kw}",
                           "front_end": f"merged linear {w.C} -> {w.J} on the tensor cores",
                           "offset_sigma_px": w.offset_sigma})
        elif isinstance(w, gen.DynWorkload):
            config.update({"H": w.H, "W": w.W, "C": w.C, "G": w.G, "kernel": f"{w.K}x{w.K}",
                           "softmax": bool(w.softmax_flag), "offsets": "none (ContMix core)"})
        elif isinstance(w, gen.DcnWorkload):
            config.update({"H": w.H, "W": w.W, "C": w.C, "G": w.G, "kernel": f"{w.kh}x{w.kw}",
                           "stride": w.stride, "pad": w.pad, "dil": w.dil,
                           "softmax": bool(w.softmax_flag), "offset_sigma_px": w.offset_sigma})
        else:
            config.update({"M": w.M, "D": w.D, "levels": [list(s) for s in w.shapes],
                           "K": w.K, "Lq": w.queries})
            if w.ref_dim:
                config.update({"reference": "box (cx, cy, w, h)" if w.ref_dim == 4 else "point",
                               "valid_ratios": "U[0.75, 1] per (image, level, axis)"})
        result = {
            "metric": metric_name(w, backward),
            "value": value,
            "unit": "taps/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": w.dtype,
            "data": "synthetic (seeded generator; no dataset or weights)",
            "config": config,
            "pixels_per_s": w.pixels() * world / (ms_per_step * 1e-3),
            "hbm_gbs": achieved,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": kernel, "algorithmic_bytes_per_launch": bytes_per_step,
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_src == "measured" else "fallback 6.65 TB/s"},
            "on_chip": (reduction_roofline(w, ms_local / args.steps, sampler, device)
                        if backward and isinstance(w, gen.DcnWorkload)
                        else fma_roofline(w, ms_local / args.steps, sampler, device)
                        if isinstance(w, gen.DynWorkload)
                        else row_gather_roofline(w, ms_local / args.steps, sampler, device)
                        if isinstance(w, gen.MsdaWorkload) and not backward
                        else on_chip_roofline(w, ms_local / args.steps, sampler, device,
                                              band=band)),
            "e2e": {"value": taps_total / (e2e_ms * 1e-3), "unit": "taps/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "steps": e2e_steps},
            "gpu_launches": int(launches),
            "clocks": sampler.summary(),
        }
        if world == 1:
            result["cpu_baseline"] = cpu_baseline(w, backward=backward, pool=pool,
                                                  cores=os.cpu_count() or 1)
    if pool is not None:
        pool.close()
        pool.join()
    if result is not None and backward:
        result["pass"] = "backward"
        result["roofline"]["note"] = (
            "timed over the whole dcn_backward / msda_backward call (zero fill, gradient "
            "kernel, rounding); algorithmic bytes = inputs + grad_out read, three "
            "gradients written once, no float32 accumulator traffic")
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()
    return result


def run_reference(args):
    """The reference arm: the float64 CPU oracle, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return None
    w = gen.WORKLOADS[args.workload]
    # size one step so that warm-up plus timed steps take about a minute
    backward = args.pass_ == "backward"
    probe = sample_of(w, 1)
    dt, taps = oracle_step(probe, seed=0, backward=backward)
    rate = taps / dt
    budget = 60.0 / max(1, args.steps + args.warmup)
    if isinstance(w, (gen.DcnWorkload, gen.DynWorkload, gen.FusedWorkload)):
        per_image = w.taps() / w.N
        n = max(1, min(w.N, int(budget * rate / per_image)))
        if budget * rate < per_image:     # less than one image: crop its rows
            rows = max(1, int(w.H * budget * rate / per_image))
            step_w = gen.scaled(w, N=1, H=rows)
        else:
            step_w = gen.scaled(w, N=n)
    else:
        per_query = w.taps() / (w.N * w.queries)
        q = max(1, min(w.queries, int(budget * rate / per_query)))
        step_w = gen.scaled(w, N=1, Lq=q)
    for i in range(args.warmup):
        oracle_step(step_w, seed=i, backward=backward)
    total_t, total_taps = 0.0, 0
    for i in range(args.steps):
        t, taps = oracle_step(step_w, seed=args.warmup + i, backward=backward)
        total_t += t
        total_taps += taps
    value = total_taps / total_t
    sample = (f"each step: oracle on {step_w.name} with N={step_w.N}"
              + (f", H={step_w.H}" if isinstance(step_w, (gen.DcnWorkload, gen.DynWorkload,
                                                             gen.FusedWorkload)) else
                 f", Lq={step_w.queries}")
              + f" ({step_w.taps()} taps), single thread, float64")
    return {
        "impl": "reference",
        "metric": metric_name(w, backward),
        "value": value,
        "unit": "taps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_t / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded generator; no dataset or weights)",
        "config": {"workload": w.name, "global_batch": w.N, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "taps/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "taps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def metric_name(w, backward):
    if backward:
        return f"backward sampled taps/s ({w.name})"
    return METRIC if w.name == gen.HEADLINE else f"sampled taps/s ({w.name})"


def torchrun_command(args, port):
    """The command that runs this benchmark as args.gpus ranks, one process
    per GPU (torch.distributed.run on this node, rendezvous on 127.0.0.1)."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
           f"--master-port={port}", os.path.abspath(__file__), "--gpus", str(args.gpus),
           "--steps", str(args.steps), "--warmup", str(args.warmup), "--impl", args.impl,
           "--workload", args.workload, "--pass", args.pass_, "--algo", args.algo]
    return cmd


def launch_ranks(args):
    """`--gpus N` without a launcher: start N ranks with torch.distributed.run
    and return its exit status.  Fails loudly when the node has fewer GPUs."""
    import socket
    import subprocess
    have = torch.cuda.device_count()
    if have < args.gpus:
        log(f"bench.py --gpus {args.gpus}: this node has {have} CUDA device(s); "
            f"{args.gpus} are needed (one rank per GPU)")
        return 2
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    return subprocess.run(torchrun_command(args, port)).returncode


def main():
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20000)
    p.add_argument("--warmup", type=int, default=200)
    p.add_argument("--impl", default="b200", choices=["b200", "reference"])
    p.add_argument("--workload", default=gen.HEADLINE, choices=sorted(gen.WORKLOADS))
    p.add_argument("--pass", dest="pass_", default="forward", choices=["forward", "backward"],
                   help="time the forward call (default) or the backward call")
    p.add_argument("--algo", default="auto", choices=["auto", "gather", "band", "simt", "tensor"],
                   help="the kernel: gather / band for the DCN forward (dcn_forward_algo), "
                        "simt / tensor for the ContMix core (dynconv_forward_algo); "
                        "auto = each call's default")
    args = p.parse_args()
    if args.warmup < 3:
        p.error("--warmup must be at least 3")
    if args.gpus < 1:
        p.error("--gpus must be at least 1")
    world = os.environ.get("WORLD_SIZE")
    if world is None and args.gpus > 1:
        sys.exit(launch_ranks(args))
    if world is not None and int(world) != args.gpus:
        p.error(f"--gpus {args.gpus} does not match the launcher's WORLD_SIZE={world}")
    result = run_reference(args) if args.impl == "reference" else run_b200(args)
    if result is not None:
        print(json.dumps(result), flush=True)


if __name__ == "__main__":
    main()
