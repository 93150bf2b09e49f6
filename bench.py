"""Benchmark of the FP8 mixed-precision training hot path on B200.

One step = one pass of the whole path over one batch of a transformer
block's four linears.  The default workload is the GPT-175B block (tokens
8192 = batch 4 x seq 2048, hidden 12288: QKV 12288->36864, out-proj
12288->12288, FFN 12288->49152->12288); `--workload gpt7b_block` runs the
GPT-7B block (tokens 4096, hidden 4096).  Per step:

  for each linear:  amax + scale + cast of X (E4M3) and dY (E5M2, mu-scaled), one
                    pass over each while its scale holds
                    fwd   Y  = Xq Wq^T     (bf16 out, fused next-amax)
                    dgrad dX = dYq Wq      (bf16 out, fused next-amax)
                    wgrad dW = dYq^T Xq    (bf16 rounded to odd, fused amax)
                    grad  gq = E5M2(mu s_g dW)
  then the precision-decoupled FP8 Adam step over the 4 weight tensors
  (E5M2 grad, E4M3 m1, FP16 m2, FP16 master; 1,811,939,328 parameters for
  GPT-175B), which also writes the E4M3 copy of each new master: the next
  step's forward and dgrad read the weight from that copy, so no weight cast
  runs in the step.  The step
  is out of place (`--adam into`, the default): each step writes the new
  state into the other of two buffer sets, in one pass while the scales
  hold; `--adam in_place` runs the in-place step (stats pass + update, the
  master's amax tracked between steps so that the stats pass skips it).

`value` is the step's algorithmic GEMM work (3 x 2MNK per linear; 89.06 TFLOP
for GPT-175B) divided by the device time of the whole step, inputs resident
in HBM.  Inputs are seeded synthetic tensors (bf16 activations ~N(0,1),
weights ~N(0,0.006) for GPT-175B / N(0,0.02) for GPT-7B, output gradients
~N(0,1e-4)); every step touches tens of GB, far more than the 126 MB L2, so no
explicit L2 flush is needed between steps.

End to end (`e2e`), each step's X and dY come from pinned host memory and
its result scalars go back; with the overlapped schedule the next step's
copy runs on a copy stream into a second buffer set while this step computes.

The step's launches run on three streams by default (--schedule overlap):
the casts of all four linears run ahead beside the GEMMs; wgrad, the
gradient cast and that tensor's Adam step run beside the next fwd/dgrad (one
Adam call per tensor instead of one over all four).  --schedule serial runs
the work in order on one stream.  The per-kernel breakdown
(`kernels`, `roofline`) always comes from a serial pass with CUDA events
around each phase.  NVTX ranges mark each linear, the Adam step and each
overlapped step for timeline profilers.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload gpt175b_block|gpt7b_block] [--schedule serial]
                    [--adam into|in_place]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from fp8_mixed_precision_tensor_b200 import synth  # noqa: E402

METRIC = "FP8 linear fwd+bwd TFLOP/s (% FP8 peak); cast & Adam GB/s (% HBM peak)"
WORKLOADS = {
    "gpt175b_block": dict(workload="gpt175b_block_linears_fp8_train_step", linears=synth.GPT175B_LINEARS,
                          tokens=synth.GPT175B_TOKENS, hidden=12288, w_std=synth.GPT175B_W_STD),
    "gpt7b_block": dict(workload="gpt7b_block_linears_fp8_train_step", linears=synth.GPT7B_LINEARS,
                        tokens=synth.GPT7B_TOKENS, hidden=4096, w_std=synth.GPT7B_W_STD),
}
MU = 2.0 ** 10
HP = dict(lr=1e-4, beta1=0.9, beta2=0.95, eps=1e-8)
# Algorithmic bytes per element / parameter (reads + writes of the definition).
CAST_BYTES_BF16 = 2 + 1       # x read once + code written (amax and cast in one pass while the scale holds)
GRAD_CAST_BYTES = 2 + 1       # round-to-odd bf16 dW read (amax fused in the GEMM) + code write
ADAM_BYTES = 11               # read g1 m1 v2 w2, write m1 v2 w2


ADAM_MODES = {
    "into": "out of place into a second set of state buffers (one pass over the state while the scales "
            "hold, a second for the chunks whose scales change)",
    "in_place": "in place (a stats pass, then the update pass)",
}


GRAD_CAST_MODES = {
    "fused": "in the out-of-place Adam pass (E5M2 codes formed in registers from the bf16 dW, never stored)",
    "separate": "a fused scale + cast kernel writing the E5M2 gradient, which Adam reads",
}


def config_of(wl: dict, schedule: str, world: int, adam: str = "into", grad_cast: str = "separate") -> dict:
    """The `config` object of the JSON line (the same for both arms)."""
    flops = sum(3 * 2 * wl["tokens"] * N * K for _, K, N in wl["linears"])
    return {"workload": wl["workload"], "tokens": wl["tokens"], "hidden": wl["hidden"],
            "linears": [l[0] for l in wl["linears"]], "adam_params": sum(N * K for _, K, N in wl["linears"]),
            "gemm_flops_per_step": flops, "l2": "inputs larger than L2 (no flush)", "schedule": schedule,
            "weight_operand": "E4M3 copy written by the previous Adam step",
            "master_amax": "tracked" if adam == "in_place" else "not tracked (no stats pass to skip)",
            "weight_gradient": "bf16 rounded to odd (its E5M2 cast equals the float32 dW's)",
            "adam_step": ADAM_MODES[adam],
            "gradient_cast": GRAD_CAST_MODES[grad_cast if adam == "into" else "separate"],
            "parallelism": f"replicas{world}" if world > 1 else "single"}


def gemm_source_digest() -> str | None:
    """sha256 of what decides the GEMM's DRAM traffic: the kernel sources
    (gemm.cuh, pipeline.cuh) and the library's GEMM launch set-up (the text
    of libfp8.cu from its tensor-map builder to the end of run_gemm, which
    picks the kernel, the tiles and the tile order).  None when that text
    cannot be found."""
    import hashlib

    csrc = os.path.join(ROOT, "fp8_mixed_precision_tensor_b200", "csrc")
    lib = open(os.path.join(csrc, "libfp8.cu"), "rb").read()
    lo, hi = lib.find(b"int make_map("), lib.find(b"void launch_amax(")
    if lo < 0 or hi < lo:
        return None
    src = b"".join(open(os.path.join(csrc, f), "rb").read() for f in ("gemm.cuh", "pipeline.cuh")) + lib[lo:hi]
    return hashlib.sha256(src).hexdigest()


def gemm_traffic(workload: str):
    """Mean DRAM bytes per GEMM launch of this step from the committed ncu
    capture, valid while the GEMM kernel source and its launch set-up (tile
    order) are the ones that were measured and the capture is of this
    workload."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "gemm_step_traffic.json")))
        digest = gemm_source_digest()
        if digest is not None and digest == rec["gemm_source_sha256"] and rec.get("workload") == workload:
            return rec["dram_bytes_per_launch_mean"]
    except Exception:
        pass
    return None


def load_peaks():
    """Measured peaks of this machine's B200s (generated file), else the
    profiling recipe's fallback.  `sus_mhz`: the median SM clock of the
    sustained measurement, when the file records one."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        p = json.load(open(path))
        sus_mhz = None
        for k, v in p.items():
            kl = k.lower()
            if "sustained" in kl and ("mhz" in kl or "clock" in kl) and isinstance(v, (int, float)):
                sus_mhz = float(v)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sus=p["bf16_tflops_sustained"],
                    sus_mhz=sus_mhz, src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, sus_mhz=1300.0, src="fallback")


def fp8_peak(peaks: dict, clocks: dict):
    """Dense FP8 peak = 2 x the bf16 peak (the nominal 4.5 / 2.25 ratio).  The
    sustained figure only when the timed region's median SM clock matches the
    clock of the sustained measurement (within 5 %); otherwise the burst
    figure, the larger one.  Returns (peak TFLOP/s, source text)."""
    mhz, mx, sus = clocks.get("sm_mhz"), clocks.get("sm_max_mhz"), peaks.get("sus_mhz")
    if mhz is not None and sus and mhz <= 1.05 * sus:
        return 2.0 * peaks["bf16_sus"], (f"2 x bf16_tflops_sustained ({peaks['src']}): median SM clock {mhz} MHz "
                                         f"matches the sustained measurement's {sus} MHz")
    return 2.0 * peaks["bf16"], (f"2 x bf16_tflops, burst ({peaks['src']}): median SM clock {mhz} MHz "
                                 f"(max {mx} MHz; sustained measurement at {sus} MHz)")


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, index: int, period_s: float = 0.02):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self.stop_ev = threading.Event()
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        names = {
            getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8): "hw_slowdown",
            getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40): "hw_thermal_slowdown",
            getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20): "sw_thermal_slowdown",
            getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4): "sw_power_cap",
            0x80: "hw_power_brake_slowdown",
        }
        while not self.stop_ev.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in names.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop_ev.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- the step
class BlockStep:
    """Device buffers and the launch sequence of one training step over a
    block's linears.  The weights exist in bf16 only at set-up: they seed the
    FP16 masters (the Adam state) and the first E4M3 weight operands; from
    then on each step's Adam writes the next step's E4M3 weights."""

    def __init__(self, device, seed: int = 0, workload: str = "gpt175b_block", adam: str = "into",
                 grad_cast: str = "separate"):
        from fp8_mixed_precision_tensor_b200 import fp8

        wl = WORKLOADS[workload]
        self.fp8 = fp8
        self.dev = device
        self.wl = wl
        self.linears = wl["linears"]
        self.M = wl["tokens"]
        f32 = dict(dtype=torch.float32, device=device)
        u8 = dict(dtype=torch.uint8, device=device)
        self.L = []
        for li, (name, K, N) in enumerate(self.linears):
            M = self.M
            d = dict(name=name, M=M, N=N, K=K)
            d["X"] = synth.device_normal((M, K), synth.ACT_STD, seed * 1000 + 10 * li + 1, torch.bfloat16, device)
            d["dY"] = synth.device_normal((M, N), synth.GRAD_STD, seed * 1000 + 10 * li + 3, torch.bfloat16, device)
            d["xq"], d["wq"], d["dyq"] = (torch.empty(s, **u8) for s in ((M, K), (N, K), (M, N)))
            d["y"] = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            d["dx"] = torch.empty((M, K), dtype=torch.bfloat16, device=device)
            # the wgrad's output, bfloat16 rounded to odd: its E5M2 cast gives the
            # codes and scale of the float32 dW's at half the bytes
            d["dw"] = torch.empty((N, K), dtype=torch.bfloat16, device=device)
            d["gq"] = torch.empty((N, K), **u8)
            # scalars: amax/scale/inv of x (0-2), w (3-5: the E4M3 weight's, rewritten by
            # Adam), dy (6-8); g scale and inverse (10, 11); fused amaxes of y, dx, dw (12-14)
            d["sc"] = torch.zeros(16, **f32)
            # Adam state: master from W (tensor-scaled FP16), zero moments, tracked master amax
            d["m"] = torch.zeros((N, K), **u8)
            d["v"] = torch.zeros((N, K), dtype=torch.int16, device=device)
            d["wh"] = torch.empty((N, K), dtype=torch.int16, device=device)
            if adam == "into":  # the out-of-place step's second state buffers
                d["m2"], d["v2"], d["wh2"] = (torch.empty_like(d[k]) for k in ("m", "v", "wh"))
            d["st"] = torch.ones(4, **f32)  # m_scale, v_scale, w_scale, tracked master amax
            d["st"][3] = -1.0
            W = synth.device_normal((N, K), wl["w_std"], seed * 1000 + 10 * li + 2, torch.bfloat16, device)
            tmp = torch.zeros(2, **f32)
            fp8.fp8_amax(W, tmp[0:1])
            fp8.fp8_scale_cast(W, fp8.FP8_F16S, tmp[0:1], 0, 1.0, d["st"][2:3], tmp[1:2], d["wh"])
            self.quantise(W, fp8.FP8_E4M3, d["sc"], 3, out=d["wq"])
            del W
            self.L.append(d)
        # Adam's chunk arrays: in place one set; out of place, step t reads the
        # state buffers of parity t % 2 (0: m, v, wh; 1: m2, v2, wh2) and writes
        # the other set
        self.adam = adam
        # the gradient cast in the Adam pass needs the out-of-place step
        self.fused_gcast = adam == "into" and grad_cast == "fused"
        sets = (("m", "v", "wh"), ("m2", "v2", "wh2")) if adam == "into" else (("m", "v", "wh"),)

        def chunk(d, k):
            # the in-place step tracks the master's amax (its stats pass then
            # skips the master); the out-of-place step has no stats pass to spare
            m, v, w = (d[x] for x in sets[k])
            g = d["dw"] if self.fused_gcast else d["gq"]
            return fp8.AdamChunk(g, d["sc"][11:12], m, d["st"][0:1], v, d["st"][1:2], w, d["st"][2:3],
                                 d["st"][3:4] if adam == "in_place" else None, d["wq"], d["sc"][4:5], d["sc"][5:6])

        def dest(d, k):
            return tuple(d[x] for x in sets[1 - k])

        self.packs, self.packs_each = [], []
        gamax = lambda ds: fp8.pack_grad_amax([d["sc"][14:15] for d in ds]) if self.fused_gcast else None
        for k in range(len(sets)):
            self.packs.append((fp8.pack_adam_chunks([chunk(d, k) for d in self.L]),
                               fp8.pack_adam_dests([dest(d, k) for d in self.L]) if adam == "into" else None,
                               gamax(self.L)))
            # one Adam call per tensor (overlapped schedule)
            self.packs_each.append([(fp8.pack_adam_chunks([chunk(d, k)]),
                                     fp8.pack_adam_dests([dest(d, k)]) if adam == "into" else None, gamax([d]))
                                    for d in self.L])
        self.ws = torch.zeros(fp8.fp8_adam_workspace_bytes(len(self.L)) // 4 + 64, **f32)
        # a 256-byte-aligned workspace slice per tensor for the per-tensor calls
        self.ws_each = torch.zeros(64 * len(self.L), **f32)
        self.t = 0
        self.flops = sum(3 * 2 * d["M"] * d["N"] * d["K"] for d in self.L)
        self.cast_elems = sum(d["M"] * d["K"] + d["M"] * d["N"] for d in self.L)
        self.params = sum(d["N"] * d["K"] for d in self.L)
        # per linear: (amax+cast pass, redo, scale) x2, 3 GEMMs, grad scale+cast;
        # Adam out of place: update, finalize, redo, finalize; in place with a
        # tracked master: stats, finalize 1, exact-master pass, finalize 2,
        # update, finalize 3
        na = 4 if adam == "into" else 6
        ng = 0 if self.fused_gcast else 1  # the gradient cast kernel
        self.launches_per_step = 4 * (2 * 3 + 3 + ng) + na
        self.launches_per_step_overlapped = 4 * (2 * 3 + 3 + ng + na)

    def adam_step(self, pack, t, ws):
        """Adam step t over the tensors of one packed (chunks, dests, gradient
        amaxes) triple."""
        chunks, dests, gamax = pack
        if self.fused_gcast:
            self.fp8.fp8_adam_step_into_castgrad(chunks, dests, gamax, MU, 0, step=t, margin=0, workspace=ws, **HP)
        elif self.adam == "into":
            self.fp8.fp8_adam_step_into(chunks, dests, step=t, margin=0, workspace=ws, **HP)
        else:
            self.fp8.fp8_adam_step(chunks, step=t, margin=0, workspace=ws, **HP)

    def quantise(self, x, fmt, sc, i, mu=1.0, out=None):
        """amax, scale and cast of x in one call: one pass over x while the
        scale (sc[i + 1], the previous step's) holds."""
        self.fp8.fp8_amax_scale_cast(x, fmt, sc[i:i + 1], 0, mu, sc[i + 1:i + 2], sc[i + 2:i + 3], out)

    def step(self, ev=None):
        """Enqueue one step on the current stream.  ev: optional dict name ->
        list of (start, end) events recorded around the GEMM / cast / Adam
        launches."""
        fp8 = self.fp8

        def mark(kind):
            if ev is None:
                return None
            e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            e[0].record()
            ev.setdefault(kind, []).append(e)
            return e

        nvtx = torch.cuda.nvtx
        for d in self.L:
            sc = d["sc"]
            nvtx.range_push(f"linear {d['name']}")
            e = mark("cast")
            self.quantise(d["X"], fp8.FP8_E4M3, sc, 0, out=d["xq"])
            self.quantise(d["dY"], fp8.FP8_E5M2, sc, 6, mu=MU, out=d["dyq"])
            if e: e[1].record()
            e = mark("gemm")
            fp8.fp8_linear_fwd(d["xq"], sc[2:3], d["wq"], sc[5:6], d["y"], sc[12:13])
            fp8.fp8_linear_dgrad(d["dyq"], sc[8:9], d["wq"], sc[5:6], d["dx"], sc[13:14])
            fp8.fp8_linear_wgrad(d["dyq"], sc[8:9], d["xq"], sc[2:3], d["dw"], sc[14:15], rto=True)
            if e: e[1].record()
            if not self.fused_gcast:
                e = mark("grad_cast")
                fp8.fp8_scale_cast(d["dw"], fp8.FP8_E5M2, sc[14:15], 0, MU, sc[10:11], sc[11:12], d["gq"])
                if e: e[1].record()
            nvtx.range_pop()
        self.t += 1
        nvtx.range_push("adam")
        e = mark("adam")
        self.adam_step(self.packs[(self.t - 1) % len(self.packs)], self.t, self.ws)
        if e: e[1].record()
        nvtx.range_pop()

    def step_overlapped(self):
        """The same work as step(), on three streams: the casts of every
        linear run ahead on a cast stream (HBM-bound work beside the
        tensor-bound GEMMs, whose CTAs leave room for a cast or Adam block per
        SM), forward and dgrad run on the current stream, wgrad, the gradient
        cast and that tensor's Adam step on an auxiliary stream (one GEMM's
        last wave overlaps the next GEMM; each tensor's optimizer step
        overlaps the following linears' GEMMs -- Adam is per tensor, so one
        call per tensor computes exactly what one call over all does).  A
        tensor's Adam rewrites its E4M3 weight, so it also waits for that
        linear's dgrad, the weight's last reader in the step.  Every buffer of
        a step is written once, and the next step's casts start only after
        this step's last Adam (the cast stream waits for an event recorded at
        the start of the next step on the current stream, which has joined the
        auxiliary stream)."""
        fp8 = self.fp8
        main = torch.cuda.current_stream()
        if not hasattr(self, "s_cast"):
            self.s_cast, self.s_aux = torch.cuda.Stream(self.dev), torch.cuda.Stream(self.dev)
            self.ev_start = torch.cuda.Event()
            self.ev_cast = [torch.cuda.Event() for _ in self.L]    # X and dY cast
            self.ev_cast_x = [torch.cuda.Event() for _ in self.L]  # X cast (enough for fwd)
            self.ev_dgrad = [torch.cuda.Event() for _ in self.L]   # the weight's last reader done
            self.ev_grad = torch.cuda.Event()
        nvtx = torch.cuda.nvtx
        nvtx.range_push("step (three streams)")
        self.ev_start.record(main)
        self.s_cast.wait_event(self.ev_start)
        self.s_aux.wait_event(self.ev_start)
        with torch.cuda.stream(self.s_cast):
            for d, e, ex in zip(self.L, self.ev_cast, self.ev_cast_x):
                sc = d["sc"]
                self.quantise(d["X"], fp8.FP8_E4M3, sc, 0, out=d["xq"])
                ex.record(self.s_cast)
                self.quantise(d["dY"], fp8.FP8_E5M2, sc, 6, mu=MU, out=d["dyq"])
                e.record(self.s_cast)
        for i, (d, e) in enumerate(zip(self.L, self.ev_cast)):
            sc = d["sc"]
            main.wait_event(self.ev_cast_x[i])
            fp8.fp8_linear_fwd(d["xq"], sc[2:3], d["wq"], sc[5:6], d["y"], sc[12:13])
            main.wait_event(e)
            fp8.fp8_linear_dgrad(d["dyq"], sc[8:9], d["wq"], sc[5:6], d["dx"], sc[13:14])
            self.ev_dgrad[i].record(main)
            self.s_aux.wait_event(e)
            with torch.cuda.stream(self.s_aux):
                fp8.fp8_linear_wgrad(d["dyq"], sc[8:9], d["xq"], sc[2:3], d["dw"], sc[14:15], rto=True)
                if not self.fused_gcast:
                    fp8.fp8_scale_cast(d["dw"], fp8.FP8_E5M2, sc[14:15], 0, MU, sc[10:11], sc[11:12], d["gq"])
                self.s_aux.wait_event(self.ev_dgrad[i])
                self.adam_step(self.packs_each[self.t % len(self.packs_each)][i], self.t + 1,
                               self.ws_each[64 * i:64 * (i + 1)])
        self.ev_grad.record(self.s_aux)
        main.wait_event(self.ev_grad)
        self.t += 1
        nvtx.range_pop()

    def result_scalars(self):
        return torch.cat([d["sc"] for d in self.L] + [d["st"] for d in self.L])


def timed_steps(runner, steps, ev=None, overlap=False):
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        if overlap:
            runner.step_overlapped()
        else:
            runner.step(ev)
    end.record()
    end.synchronize()
    return start.elapsed_time(end)


def sum_events(ev, kind):
    return sum(a.elapsed_time(b) for a, b in ev.get(kind, []))


# ---------------------------------------------------------------- CPU oracle timing
class OracleSample:
    """A bounded sample of one step's work for the CPU oracle: per linear the
    forward GEMM of one token row against the whole weight (dgrad and wgrad
    have the same multiply-add count, so the row's time counts three
    times), an amax + scale + cast of 2^21 bf16 elements and an Adam step on
    2^20 parameters.  Inputs are drawn once; run() times one sample and
    returns (seconds of the sample, seconds extrapolated to the whole step by
    units)."""

    ROWS = 1

    def __init__(self, wl: dict):
        import oracle

        self.oracle = oracle
        self.wl = wl
        self.ops = []
        for name, K, N in wl["linears"]:
            g = synth.rng("bench-oracle", name)
            # finite positive E4M3 codes (bit 3 clear: never 0x7F)
            wq = (np.frombuffer(g.bytes(N * K), dtype=np.uint8) & 0x77).reshape(N, K)
            xq = (np.frombuffer(g.bytes(self.ROWS * K), dtype=np.uint8) & 0x77).reshape(self.ROWS, K)
            self.ops.append((name, K, N, xq, wq))
        self.n_cast = 1 << 21
        self.xb = synth.normal_bf16((self.n_cast,), 1.0, "bench-oracle", "cast")
        self.n_adam = 1 << 20
        self.gq = np.random.default_rng(0).integers(0, 0x7B, self.n_adam, dtype=np.uint8)
        M = wl["tokens"]
        self.elems = sum(M * K + M * N for _, K, N in wl["linears"])  # X and dY casts
        self.params = sum(N * K for _, K, N in wl["linears"])
        self.cores = oracle.num_threads()
        self.text = (f"oracle timed on: per linear a {self.ROWS}-row forward GEMM block "
                     f"({'; '.join(f'{n}: {self.ROWS}x{N}x{K}' for n, K, N, _, _ in self.ops)}), counted "
                     f"x3 for dgrad/wgrad; amax+scale+cast of 2^21 bf16; Adam on 2^20 params; "
                     f"extrapolated to the full step by units")

    def run(self):
        o = self.oracle
        M = self.wl["tokens"]
        t_sample = 0.0
        t_full = 0.0
        for name, K, N, xq, wq in self.ops:
            t0 = time.perf_counter()
            o.linear_fwd(xq, 1.0, wq, 1.0, self.ROWS, N, K)
            dt = time.perf_counter() - t0
            t_sample += dt
            t_full += 3 * dt * M / self.ROWS
        t0 = time.perf_counter()
        a = o.amax(self.xb, o.DT_BF16, parallel=True)
        _, s = o.compute_scale(a, o.E4M3, 0)
        o.cast(self.xb, o.E4M3, s, o.DT_BF16)
        dt = time.perf_counter() - t0
        t_sample += dt
        t_full += dt / self.n_cast * (self.elems + self.params)  # X/dY casts + gradient cast
        n = self.n_adam
        t0 = time.perf_counter()
        o.adam_step(self.gq, 1e-6, np.zeros(n, np.uint8), 1.0, np.zeros(n, np.uint16), 1.0,
                    np.full(n, 0x2C00, np.uint16), 1.0, t=1, margin=0, **HP)
        dt = time.perf_counter() - t0
        t_sample += dt
        t_full += dt / n * self.params
        return t_sample, t_full


# ---------------------------------------------------------------- arms
def run_reference(args):
    """The CPU oracle as it stands, on the host cores: each step is one
    bounded sample of the step's work (OracleSample); `ms_per_step` is the
    measured time of one such sample, `value` the GEMM work of the whole
    step over the time extrapolated from the sample by units."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    cfg = config_of(wl, args.schedule, args.gpus, args.adam, args.grad_cast)
    sample = OracleSample(wl)
    t_s, t_f = [], []
    for i in range(args.warmup + args.steps):
        a, b = sample.run()
        if i >= args.warmup:
            t_s.append(a)
            t_f.append(b)
    ts, tf = statistics.median(t_s), statistics.median(t_f)
    v = cfg["gemm_flops_per_step"] / tf / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ts * 1e3,
            "ms_per_full_step_extrapolated": tf * 1e3, "extrapolated": True, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": sample.cores, "kind": "oracle",
                             "sample": sample.text},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_gpu(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    from fp8_mixed_precision_tensor_b200 import fp8

    peaks = load_peaks()
    wl = WORKLOADS[args.workload]
    runner = BlockStep(dev, seed=rank, workload=args.workload, adam=args.adam, grad_cast=args.grad_cast)
    overlap = args.schedule == "overlap"
    for _ in range(args.warmup):
        runner.step_overlapped() if overlap else runner.step()
    barrier()

    # ---- device-timed region: inputs resident, whole step
    sampler = ClockSampler(local)
    with sampler:
        barrier()
        ms = timed_steps(runner, args.steps, overlap=overlap)
        barrier()
    ms_step = ms / args.steps
    if dist is not None:
        t = torch.tensor([ms_step], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step = t.item()
    status = fp8.fp8_get_status()
    clocks = sampler.summary()

    # ---- per-kernel breakdown (separate pass with events between phases)
    ev = {}
    timed_steps(runner, args.steps, ev)
    t_gemm = sum_events(ev, "gemm") / args.steps
    t_cast = sum_events(ev, "cast") / args.steps
    t_gcast = sum_events(ev, "grad_cast") / args.steps
    t_adam = sum_events(ev, "adam") / args.steps

    # ---- end to end: host inputs (pinned) copied in, result scalars read back
    host_in = [(d["X"].cpu().pin_memory(), d["dY"].cpu().pin_memory()) for d in runner.L]
    res = torch.empty(runner.result_scalars().numel(), dtype=torch.float32).pin_memory()
    h2d = sum(x.numel() * x.element_size() + y.numel() * y.element_size() for x, y in host_in)
    d2h = res.numel() * 4

    def e2e_step():
        for d, (x, y) in zip(runner.L, host_in):
            d["X"].copy_(x, non_blocking=True)
            d["dY"].copy_(y, non_blocking=True)
        runner.step()
        res.copy_(runner.result_scalars(), non_blocking=True)

    # Overlapped schedule: the inputs of step t+1 are copied on a copy stream
    # into a second set of device buffers while step t computes (prefetching
    # input pipeline); every step's copy is still inside the timed region.
    sets = ([[(d["X"], d["dY"]) for d in runner.L],
             [(torch.empty_like(d["X"]), torch.empty_like(d["dY"])) for d in runner.L]] if overlap else None)
    copy_stream = torch.cuda.Stream(dev)
    ev_copied = [torch.cuda.Event(), torch.cuda.Event()]
    ev_used = [torch.cuda.Event(), torch.cuda.Event()]

    def copy_into(k):
        copy_stream.wait_event(ev_used[k])  # the steps that read set k have cast it
        with torch.cuda.stream(copy_stream):
            for (xd, yd), (x, y) in zip(sets[k], host_in):
                xd.copy_(x, non_blocking=True)
                yd.copy_(y, non_blocking=True)
        ev_copied[k].record(copy_stream)

    def e2e_steps_pipelined(steps):
        main = torch.cuda.current_stream()
        for k in range(2):
            ev_used[k].record(main)
        copy_into(0)
        for t in range(steps):
            cur = t % 2
            if t + 1 < steps:
                copy_into(1 - cur)
            main.wait_event(ev_copied[cur])
            for d, (xd, yd) in zip(runner.L, sets[cur]):
                d["X"], d["dY"] = xd, yd
            runner.step_overlapped()
            ev_used[cur].record(runner.s_cast)
            res.copy_(runner.result_scalars(), non_blocking=True)
        main.wait_stream(copy_stream)

    if overlap:
        e2e_steps_pipelined(2)
    else:
        for _ in range(2):
            e2e_step()
    barrier()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    if overlap:
        e2e_steps_pipelined(args.steps)
    else:
        for _ in range(args.steps):
            e2e_step()
    s1.record()
    s1.synchronize()
    e2e_ms = s0.elapsed_time(s1) / args.steps
    if overlap:
        for d, (xd, yd) in zip(runner.L, sets[0]):
            d["X"], d["dY"] = xd, yd
    if dist is not None:
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = t.item()
    status |= fp8.fp8_get_status()

    value = runner.flops * world / (ms_step * 1e-3) / 1e12
    peak, peak_src = fp8_peak(peaks, clocks)
    gemm_tflops = runner.flops / (t_gemm * 1e-3) / 1e12
    cast_gbs = runner.cast_elems * CAST_BYTES_BF16 / (t_cast * 1e-3) / 1e9
    gcast_gbs = runner.params * GRAD_CAST_BYTES / (t_gcast * 1e-3) / 1e9 if t_gcast > 0 else None
    # with the gradient cast in the pass, Adam reads the bf16 dW (2 B) instead of the E5M2 code
    adam_bytes = ADAM_BYTES + (1 if runner.fused_gcast else 0)
    adam_gbs = runner.params * adam_bytes / (t_adam * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8(e4m3/e5m2)->f32 accum; f32 elementwise", "data": "synthetic",
        "config": config_of(wl, args.schedule, world, args.adam, args.grad_cast),
        "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": gemm_tflops / peak, "traffic": gemm_traffic(wl["workload"]),
                     "kernel": "k_gemm3 (fwd+dgrad+wgrad; achieved = GEMM flops per step / summed GEMM "
                               "time; traffic = mean DRAM bytes per launch)",
                     "peak_src": peak_src},
        "kernels": {
            "gemm": {"ms": t_gemm, "TFLOP/s": gemm_tflops, "frac_fp8_peak": gemm_tflops / peak},
            "amax_scale_cast": {"ms": t_cast, "GB/s": cast_gbs, "frac_hbm": cast_gbs / peaks["hbm"],
                                "tensors": "X and dY of every linear (the weight operand comes from Adam)"},
            "grad_cast": ({"ms": t_gcast, "GB/s": gcast_gbs, "frac_hbm": gcast_gbs / peaks["hbm"]}
                          if gcast_gbs is not None else {"ms": 0.0, "fused": "in the Adam pass"}),
            "adam": {"ms": t_adam, "GB/s": adam_gbs, "frac_hbm": adam_gbs / peaks["hbm"],
                     "bytes_per_param_algorithmic": adam_bytes,
                     "bytes_per_param_moved": ("11 (one pass while the scales hold; 22 for a chunk whose "
                                               "scales change) + 1 for the E4M3 weight copy"
                                               if args.adam == "into" else
                                               "15 (stats pass 4 with the tracked master + update 11) "
                                               "+ 1 for the E4M3 weight copy")},
            "hbm_peak_gbs": peaks["hbm"],
        },
        "e2e": {"value": runner.flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": (runner.launches_per_step_overlapped if overlap else runner.launches_per_step) * args.steps,
        "clocks": clocks,
        "device_status": status,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = OracleSample(wl)
        runs = [sample.run() for _ in range(2)]
        t_cpu = statistics.median(r[1] for r in runs)
        line["cpu_baseline"] = {"value": runner.flops / t_cpu / 1e12, "unit": "TFLOP/s", "cores": sample.cores,
                                "kind": "oracle", "sample": sample.text,
                                "sample_seconds": statistics.median(r[0] for r in runs)}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gpt175b_block", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--schedule", default="overlap", choices=["overlap", "serial"],
                    help="overlap: casts / GEMMs / wgrad on three streams; serial: one stream")
    ap.add_argument("--grad-cast", dest="grad_cast", default="separate", choices=sorted(GRAD_CAST_MODES),
                    help="separate: the E5M2 gradient cast as its own kernel; fused: inside the out-of-place "
                         "Adam pass (fewer bytes, but measured 0.3-0.4 ms slower in the overlapped step)")
    ap.add_argument("--adam", default="into", choices=sorted(ADAM_MODES),
                    help="into: out-of-place Adam step (two state buffers); in_place: stats + update passes")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
