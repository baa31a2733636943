#!/usr/bin/env python
"""Throughput of the group-limited routed MoE layer (Ling-3.0-tiny shapes) on B200.

One step = one whole layer (route -> permute -> gate/up GEMM -> down GEMM ->
combine) through the C ABI on one batch of seeded synthetic tokens that are
already resident in HBM.  The headline workload is the long-prompt prefill
(8,189 real tokens in buffers of 8,192); the decode batch of 16 tokens is
measured the same way and reported beside it.

Timing: W warm-up steps, then exactly K timed steps between a barrier and a
device synchronize.  A step is one moe_layer call (the public layer API; a
workspace allocated once).  Before every step a 256 MB buffer is overwritten
and another 256 MB read, so that L2 holds neither the inputs nor dirty lines,
and a short device-side sleep lets the host enqueue the whole step before the
GPU reaches it (all outside the step's events).  Each step is bracketed by one
pair of CUDA events on the launching stream, with nothing between its
launches, so programmatic dependent launch overlaps each kernel's prologue
with its predecessor's tail as in any real run.  The per-kernel breakdown and
the dominant kernel's roofline come from a second pass of K steps over the
same batch through the five step calls, with events between them.  The
decode batch is also timed as a replayed CUDA graph of the moe_layer call.
The end-to-end figure (`e2e`) goes through the public host-buffer API
(moe.HostPipeline over the C ABI's moe_layer_host): every step copies its own x and
router logits in and its output out, with two steps in flight on two streams
so that copies and layers overlap.
Multi-GPU (torchrun): every rank runs its own independent batch (data-parallel
replicas, weak scaling, no data-path collective); the reported time is the
max over ranks.

``--impl reference`` times the float64 CPU oracle instead (rank 0 only).
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
sys.path.insert(0, ROOT)

from group_limited_routed_moe_b200 import synth  # noqa: E402

GATE_UP_BYTES_PER_EXPERT = 2 * 1536 * 512 * 2
DOWN_BYTES_PER_EXPERT = 1536 * 512 * 2
# block-FP8 expert: one byte per weight, one fp32 scale per 128 x 128 block
FP8_BYTES_PER_EXPERT = 3 * 1536 * 512 + (2 * 12 * 4 + 4 * 12) * 4
# NVFP4 expert in its checkpoint form: half a byte per weight, one E4M3 byte per
# 16 weights (the three fp32 tensor scales are negligible)
NVFP4_BYTES_PER_EXPERT = 3 * 1536 * 512 // 2 + 3 * 1536 * 512 // 16
# what the NVFP4 kernel streams: codes, and a 16-bit multiplier per 16 weights
NVFP4_PACKED_BYTES_PER_EXPERT = 3 * 1536 * 512 // 2 + 3 * 1536 * 512 // 16 * 2
FLOPS_PER_ROW = 2 * (1536 * 1024 + 512 * 1536)          # one (token, expert) pair
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_T8189", choices=["prefill_T8189", "decode_T16"])
    ap.add_argument("--weights", default="bf16", choices=["bf16", "fp8", "nvfp4"],
                    help="expert weights of the main line: bf16, block FP8 (E4M3 codes, "
                         "power-of-two 128x128 block scales) or NVFP4 (E2M1 codes, E4M3 "
                         "scales per 16, power-of-two tensor scales)")
    ap.add_argument("--e256-prefill", action="store_true",
                    help="also time the 256-expert shape at T=8189 (secondary line)")
    ap.add_argument("--shared", type=int, default=0,
                    help="shared experts (0-8) added to the main line's layer")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the decode_T16 (bf16, FP8, NVFP4, shared-expert) measurements")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the decode_T4 (seeds 1-8) and prefill_T2048_skewed lines")
    ap.add_argument("--no-stack", action="store_true",
                    help="skip the 23-layer stack lines (T=1 and T=8189, one CUDA graph each)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample", type=int, default=2048, help="tokens in the oracle sample")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# The sources each profiled expert-FFN kernel is built from: the wide
# (tokens-as-M) kernel of batches above 256 tokens, and the skinny
# (weights-as-M) kernel of smaller ones with its bf16, FP8 and NVFP4 forms.
WIDE_SOURCES = ("common.cuh", "expert_ffn.cuh")
SKINNY_SOURCES = ("common.cuh", "expert_ffn.cuh", "expert_ffn_skinny.cuh", "fp8.cuh", "fp4.cuh",
                  "pack.cuh", "combine.cuh")
# Up to this many tokens the expert-FFN launch of a layer also runs its combine
# (kFusedCombineMaxT in csrc/combine.cuh), except beside a separate
# shared-expert launch (quantised routed experts with shared experts).
FUSED_COMBINE_MAX_T = 1


def kernel_sources(workload: str):
    return WIDE_SOURCES if synth.WORKLOADS[workload].T > 256 else SKINNY_SOURCES


def kernel_source_sha(files):
    """sha256 (first 16 hex digits) of the given kernel sources, concatenated
    in order: what a profile's counters are valid for."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "group_limited_routed_moe_b200", "csrc")
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch from the committed ncu summary, if it
    was taken on the current sources of that workload's kernel; else None."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(p):
        return None
    sha, traffic = None, None
    for line in open(p):
        if line.startswith("source_sha:"):
            sha = line.split(":", 1)[1].strip()
        if line.startswith("traffic_bytes_per_launch:"):
            traffic = float(line.split(":", 1)[1].strip())
    return traffic if sha == kernel_source_sha(kernel_sources(workload)) else None


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML every few ms."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int):
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover
            self.err = str(e)
        self.samples, self.reasons = [], 0
        self._stop = threading.Event()

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self._sample()  # the thread may get few turns while the host enqueues
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._sample()
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and b != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": names}


# --------------------------------------------------------------------- our arm

class LayerRun:
    """Device buffers and the five-call step of one workload."""

    def __init__(self, wl: synth.Workload, dev, weights, fp8: bool = False, shared=None,
                 nvfp4: bool = False):
        import torch
        from group_limited_routed_moe_b200 import moe
        self.moe, self.torch, self.wl, self.dev = moe, torch, wl, dev
        self.fp8 = fp8  # weights: a packed block-FP8 layer (moe_layer_fp8)
        self.nvfp4 = nvfp4  # weights: a packed NVFP4 layer (moe_layer_nvfp4)
        quant = fp8 or nvfp4
        self.shared = shared  # None, or (packed shared experts, n_shared): moe_layer_shared
        self.T = wl.T
        tok = synth.make_tokens(wl.T, wl.seed, hot=wl.hot)
        self.tok = tok
        T, Tb = wl.T, wl.T_buf
        bf = torch.bfloat16
        self.x = torch.zeros((Tb, 1536), dtype=bf, device=dev)
        self.x[:T] = torch.from_numpy(tok.x_bits.view(np.int16)).to(dev).view(bf)
        self.logits = torch.zeros((Tb, 128), dtype=torch.float32, device=dev)
        self.logits[:T] = torch.from_numpy(tok.logits).to(dev)
        self.bias = torch.from_numpy(tok.bias).to(dev)
        self.packed = weights
        n = T * 8
        i32 = torch.int32
        self.idx = torch.empty((T, 8), dtype=i32, device=dev)
        self.w = torch.empty((T, 8), dtype=torch.float32, device=dev)
        self.counts = torch.empty(128, dtype=i32, device=dev)
        self.offsets = torch.empty(moe.OFFSETS_LEN, dtype=i32, device=dev)
        self.perm_src = torch.empty(n, dtype=i32, device=dev)
        self.inv_perm = torch.empty(n, dtype=i32, device=dev)
        wsb = moe.permute_workspace_bytes(T)
        self.pws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev) if wsb else None
        self.h = torch.empty((n, 512), dtype=torch.float16, device=dev)
        self.y = torch.empty((n, 1536), dtype=torch.float16, device=dev)
        self.out = torch.empty((Tb, 1536), dtype=bf, device=dev)
        # moe_layer launches: route + permute (one fused kernel up to 64 tokens;
        # route and one permute kernel up to 1024; route, count and fused scan/scatter
        # up to 256 blocks of 128 tokens; route, count, scan, scatter beyond), the
        # expert FFN (gate/up and down in one launch), combine (inside the FFN
        # launch up to FUSED_COMBINE_MAX_T tokens)
        nb = (T + 127) // 128
        n_rp = 1 if T <= 64 else 2 if T <= 1024 else (3 if nb <= 256 else 4)
        fused = T <= FUSED_COMBINE_MAX_T and not (quant and shared is not None)
        self.launches_per_step = n_rp + 1 + (0 if fused else 1)
        fws = moe.lib.moe_expert_ffn_fp8_workspace_bytes(T) if quant else 0
        self.ffn_ws = torch.empty(fws, dtype=torch.uint8, device=dev) if fws else None
        if fws:
            self.launches_per_step += 1  # FP8 / NVFP4 above 256 tokens: the expansion pass
        # the breakdown pass times the same kernels the layer call runs
        self.part_names = ["route", "permute", "expert_ffn", "combine"]
        self.lws = moe.alloc_layer_workspace(T, dev, fp8=quant)
        if shared is not None:
            n = moe.layer_shared_workspace_bytes(T, shared[1], quant)
            raw = torch.empty(n + 1024, dtype=torch.uint8, device=dev)
            off = (-raw.data_ptr()) % 1024
            self.lws = raw[off:off + n]
            # the shared row set; with quantised routed experts also the shared
            # experts' own FFN launch (bf16: a second segment of the routed launch)
            self.launches_per_step += 2 if quant else 1
        self.flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.read_buf = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
        self.write_only_flush = False
        self.stream = torch.cuda.current_stream()

    def flush(self, prime=True):
        # Overwrite 256 MB (evicts every line of the step's inputs from the 126 MB
        # L2), then read another 256 MB so that the dirty lines of that write are
        # written back here rather than inside the first kernel of the step.
        self.flush_buf.fill_(1)
        if not self.write_only_flush:
            self.read_buf.max()
        if prime:  # ~0.5 ms spin so that the five launches are queued before the GPU gets there
            self.torch.cuda._sleep(1_000_000)

    def step(self):
        """One layer through the public layer call (what a user runs)."""
        if self.shared is not None:
            kw = ({"packed_nvfp4": self.packed} if self.nvfp4 else
                  {"packed_fp8": self.packed} if self.fp8 else {"packed_w": self.packed})
            self.moe.moe_layer_shared(self.x[:self.T], self.logits[:self.T], self.bias,
                                      self.shared[0], self.shared[1], out=self.out[:self.T],
                                      workspace=self.lws, stream=self.stream, **kw)
            return
        self.layer_fn(self.x[:self.T], self.logits[:self.T], self.bias, self.packed,
                      out=self.out[:self.T], workspace=self.lws, stream=self.stream)

    @property
    def layer_fn(self):
        m = self.moe
        return m.moe_layer_nvfp4 if self.nvfp4 else m.moe_layer_fp8 if self.fp8 else m.moe_layer

    def step_parts(self, ev):
        """The same layer through the step calls, with an event between each."""
        m, T, s = self.moe, self.T, self.stream
        k = iter(range(len(ev)))
        rec = lambda: ev[next(k)].record(s)  # noqa: E731
        rec()
        m.moe_route(self.logits[:T], self.bias, self.idx, self.w, stream=s)
        rec()
        m.moe_permute(self.idx, self.counts, self.offsets, self.perm_src, self.inv_perm,
                      self.pws, stream=s)
        rec()
        if self.fp8 or self.nvfp4:
            (m.moe_expert_ffn_nvfp4 if self.nvfp4 else m.moe_expert_ffn_fp8)(
                self.x[:T], self.packed, self.offsets, self.perm_src, self.h, self.y,
                workspace=self.ffn_ws, stream=s)
        else:
            m.moe_expert_ffn(self.x[:T], self.packed, self.offsets, self.perm_src, self.h,
                             self.y, stream=s)
        rec()
        m.moe_combine(self.y, self.w, self.inv_perm, out=self.out[:T], stream=s)
        rec()

    def timed(self, steps, warmup, barrier):
        """K whole steps, each between one pair of events; returns ms per step."""
        torch = self.torch
        for _ in range(warmup):
            self.flush()
            self.step()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        s = self.stream
        barrier()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for k in range(steps):
            self.flush()
            evs[k][0].record(s)
            self.step()
            evs[k][1].record(s)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
        barrier()
        return np.array([e[0].elapsed_time(e[1]) for e in evs]), wall

    def router(self, steps, peaks):
        """The router projection (moe_router) alone on this batch: K launches after
        the same L2 flush, against the HBM roofline (x, W_router and the logits
        cross HBM once; 2 flop per byte of x per expert is far below the ridge)."""
        torch, moe = self.torch, self.moe
        T = self.T
        w_bits = synth.router_weight_bits_np(0, 0)
        w = torch.from_numpy(w_bits.view(np.int16)).to(self.dev).view(torch.bfloat16)
        packed = moe.moe_pack_router(w)
        logits = torch.empty((T, 128), dtype=torch.float32, device=self.dev)
        moe.moe_router(self.x[:T], packed, logits)
        times = []
        for _ in range(steps):
            self.flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(self.stream)
            moe.moe_router(self.x[:T], packed, logits, stream=self.stream)
            b.record(self.stream)
            times.append((a, b))
        torch.cuda.synchronize()
        us = float(np.mean([a.elapsed_time(b) for a, b in times])) * 1e3
        nbytes = T * 1536 * 2 + 1536 * 128 * 2 + T * 128 * 4
        achieved = nbytes / (us * 1e-6) / 1e9
        peak = float(peaks["hbm_gbs"])
        return {"kernel": "router_kernel (logits = x W_router, tcgen05)", "us": round(us, 2),
                "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "algorithmic_per_launch": nbytes,
                "flops_per_launch": 2 * T * 1536 * 128}

    def dirty_l2_steps(self, steps, barrier):
        """Context only: the same K steps after a write-only flush, which leaves
        about 126 MB of dirty lines in L2 for the step's first kernels to write
        back.  Mean ms per step."""
        self.write_only_flush = True
        try:
            st, _ = self.timed(steps, 2, barrier)
        finally:
            self.write_only_flush = False
        return float(st.mean())

    def breakdown(self, steps):
        """K more steps with events between the step calls: ms [K][parts]."""
        torch = self.torch
        n = len(self.part_names)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
        torch.cuda.synchronize()
        for k in range(steps):
            self.flush()
            self.step_parts(evs[k])
        torch.cuda.synchronize()
        return np.array([[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(n)]
                         for k in range(steps)])

    def graph_layer_us(self, steps, warmup):
        """The fused moe_layer call captured once in a CUDA graph and replayed."""
        torch, moe = self.torch, self.moe
        T = self.T
        ws = moe.alloc_layer_workspace(T, self.dev, fp8=self.fp8 or self.nvfp4)
        layer = self.layer_fn
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            layer(self.x[:T], self.logits[:T], self.bias, self.packed, out=self.out[:T],
                  workspace=ws, stream=s)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                layer(self.x[:T], self.logits[:T], self.bias, self.packed, out=self.out[:T],
                      workspace=ws, stream=s)
        torch.cuda.synchronize()
        cur = torch.cuda.current_stream()
        for _ in range(warmup):
            self.flush(prime=False)
            g.replay()
        times = []
        for _ in range(steps):
            self.flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(cur)
            g.replay()
            b.record(cur)
            times.append((a, b))
        torch.cuda.synchronize()
        del g
        return float(np.mean([a.elapsed_time(b) for a, b in times])) * 1e3

    def e2e(self, steps, warmup, depth=3):
        """The layer end to end through the public API from pinned host buffers:
        every step copies its x and router logits host -> device, runs the layer
        and copies its output device -> host.  Steps go through a HostPipeline
        with `depth` in flight, so one step's copies overlap another's layer.
        Returns (ms per step over K steps, bytes host->device and device->host
        per step).  No flush between steps: every step streams the touched
        experts' weights, far more than L2 holds."""
        torch, moe = self.torch, self.moe
        T = self.T
        x_h = torch.from_numpy(self.tok.x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
        lg_h = torch.from_numpy(self.tok.logits).pin_memory()
        outs_h = [torch.empty((T, 1536), dtype=torch.bfloat16).pin_memory() for _ in range(depth)]
        pipe = moe.HostPipeline(T, self.dev, depth, fp8=self.fp8, shared=self.shared,
                                nvfp4=self.nvfp4)

        def run(n):
            for k in range(n):
                pipe.submit(x_h, lg_h, outs_h[k % depth], self.bias, self.packed)
        run(warmup)
        pipe.drain()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cur = torch.cuda.current_stream()
        a.record(cur)
        for st in pipe.streams():
            st.wait_event(a)
        run(steps)
        for st in pipe.streams():
            ev = torch.cuda.Event()
            ev.record(st)
            cur.wait_event(ev)
        b.record(cur)
        b.synchronize()
        # the last output is the one each slot produced last: check it arrived
        assert torch.equal(outs_h[(steps - 1) % depth].view(torch.int16),
                           self.out[:T].cpu().view(torch.int16))
        return a.elapsed_time(b) / steps, x_h.numel() * 2 + lg_h.numel() * 4, outs_h[0].numel() * 2


def max_over_ranks(value: float, dist, device) -> float:
    """The largest of every rank's `value` (each rank's own when dist is None)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank's batch over the slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step * 1e-3)


def distinct_experts(run):
    """Experts with at least one row in the timed steps (the permute's counts)."""
    return int((run.counts > 0).sum().item())


def roofline_for(wl, run, per_ms, peaks, peak_kind):
    """Roofline of the dominant kernel of one workload: the expert FFN launch
    (gate/up + SwiGLU + down).  Prefill-sized batches are bound by the tensor
    cores (both GEMMs' flops), decode-sized ones by HBM (the touched experts'
    weights, x read, y_perm written)."""
    T = wl.T
    ffn_ms = float(per_ms[:, run.part_names.index("expert_ffn")].mean())
    if run.nvfp4 and T <= 256:
        # NVFP4 codes and block scales of the touched experts in the checkpoint's form
        # (the kernel reads 16-bit multipliers in place of the 8-bit scales: see
        # "streamed_per_launch"), x read, y_perm written
        d = distinct_experts(run)
        act = T * 1536 * 2 + 8 * T * 1536 * 2
        nbytes = d * NVFP4_BYTES_PER_EXPERT + act
        peak = float(peaks["hbm_gbs"])
        achieved = nbytes / (ffn_ms * 1e-3) / 1e9
        return {"kernel": "skinny_gemm_kernel<3, 2> (E2M1 codes dequantised into tensor memory; "
                          "gate/up + SwiGLU + down in one launch)",
                "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
                "algorithmic_per_launch": nbytes,
                "streamed_per_launch": d * NVFP4_PACKED_BYTES_PER_EXPERT + act,
                "distinct_experts": d,
                "traffic": profiled_traffic("expert_ffn_nvfp4", wl.name)}
    if run.fp8 and T <= 256:
        # block-FP8 codes and scales of the touched experts, x read, y_perm written
        d = distinct_experts(run)
        nbytes = d * FP8_BYTES_PER_EXPERT + T * 1536 * 2 + 8 * T * 1536 * 2
        peak = float(peaks["hbm_gbs"])
        achieved = nbytes / (ffn_ms * 1e-3) / 1e9
        return {"kernel": "skinny_gemm_kernel<3, fp8> (E4M3 codes dequantised in shared memory; "
                          "gate/up + SwiGLU + down in one launch)",
                "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
                "algorithmic_per_launch": nbytes, "distinct_experts": d,
                "traffic": profiled_traffic("expert_ffn_fp8", wl.name)}
    if T >= 2048:
        flops = FLOPS_PER_ROW * 8 * T
        key = "bf16_tflops"
        peak = float(peaks[key])
        achieved = flops / (ffn_ms * 1e-3) / 1e12
        kernel = "ffn_gemm_kernel<3> (gate/up + SwiGLU + down in one launch)"
        if run.fp8 or run.nvfp4:
            kernel = ("dequant_fp4_kernel + " if run.nvfp4 else "dequant_fp8_kernel + ") + \
                kernel + ", timed together"
        return {"kernel": kernel,
                "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_kind} {key} (burst)", "algorithmic_per_launch": flops,
                "traffic": None if run.fp8 or run.nvfp4 else profiled_traffic("expert_ffn", wl.name)}
    d = distinct_experts(run)
    nbytes = (d * (GATE_UP_BYTES_PER_EXPERT + DOWN_BYTES_PER_EXPERT) + T * 1536 * 2
              + 8 * T * 1536 * 2)
    peak = float(peaks["hbm_gbs"])
    achieved = nbytes / (ffn_ms * 1e-3) / 1e9
    kernel = ("skinny_gemm_kernel<3>" if T <= 256 else "ffn_gemm_kernel<3>") + \
        " (gate/up + SwiGLU + down in one launch)"
    return {"kernel": kernel, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
            "unit": "GB/s", "frac": round(achieved / peak, 4),
            "peak_source": f"{peak_kind} hbm_gbs", "algorithmic_per_launch": nbytes,
            "distinct_experts": d, "traffic": profiled_traffic("expert_ffn", wl.name)}


def layer_fractions(wl, run, step_ms, per_ms, peaks):
    """Whole-layer fractions (context): tokens/s against the HBM bound of the
    distinct experts' weights and against the tensor bound of the useful flops."""
    layer_s = float(step_ms.mean()) * 1e-3
    d = distinct_experts(run)
    per_expert = (NVFP4_BYTES_PER_EXPERT if run.nvfp4 else FP8_BYTES_PER_EXPERT if run.fp8
                  else GATE_UP_BYTES_PER_EXPERT + DOWN_BYTES_PER_EXPERT)
    nbytes = d * per_expert + wl.T * (1536 * 4 + 512)
    flops = FLOPS_PER_ROW * 8 * wl.T
    return {"layer_us": round(layer_s * 1e6, 2),
            "hbm_frac": round(nbytes / layer_s / 1e9 / float(peaks["hbm_gbs"]), 4),
            "tensor_frac": round(flops / layer_s / 1e12 / float(peaks["bf16_tflops"]), 4),
            "kernel_us": {k: round(float(per_ms[:, i].mean()) * 1e3, 2) for i, k in
                          enumerate(run.part_names)},
            "kernel_us_sum": round(float(per_ms.sum(axis=1).mean()) * 1e3, 2),
            "distinct_experts": d}


def cpu_baseline(wl, tok, host_w, sample, fp8=False, nvfp4=False):
    """The float64 oracle on the first `sample` tokens.  host_w: bf16 bits
    (W_gate, W_up, W_down), or with fp8 the codes and scales (q_gate, s_gate,
    q_up, s_up, q_down, s_down), or with nvfp4 the codes, block and tensor
    scales of each matrix."""
    import oracle as O
    from threadpoolctl import threadpool_info
    n = min(sample, wl.T)
    rows = np.arange(n)
    t0 = time.perf_counter()
    fn = O.moe_layer_nvfp4 if nvfp4 else O.moe_layer_fp8 if fp8 else O.moe_layer
    fn(tok.x_bits[rows], tok.logits[rows], tok.bias, *host_w)
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {"value": round(n / dt, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": (f"first {n} of {wl.T} tokens of {wl.name}"
                       f"{' (NVFP4 experts)' if nvfp4 else ' (block-FP8 experts)' if fp8 else ''}"
                       f", float64 NumPy oracle, {dt:.2f} s")}


def decode_line(wl2, dev, packed, fp8, steps, warmup, peaks, peak_kind, barrier, nvfp4=False):
    """The decode batch measured beside the main line: whole-layer steps,
    breakdown and roofline, router, CUDA-graph replay, end to end."""
    run2 = LayerRun(wl2, dev, packed, fp8=fp8, nvfp4=nvfp4)
    clk2 = ClockSampler(int(dev.index or 0))
    n = max(steps, 50)
    with clk2:
        steps2, _ = run2.timed(n, warmup, barrier)
    per2 = run2.breakdown(n)
    dirty2 = run2.dirty_l2_steps(n, barrier)
    e2e2, h2d2, d2h2 = run2.e2e(40, 3)
    graph_us = run2.graph_layer_us(50, 3)
    ms2 = float(steps2.mean())
    out = {
        "value": round(wl2.T / (ms2 * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(ms2, 5),
        "roofline": roofline_for(wl2, run2, per2, peaks, peak_kind)}
    if not (fp8 or nvfp4):
        out["router"] = run2.router(20, peaks)
    out.update({
        "layer": dict(layer_fractions(wl2, run2, steps2, per2, peaks),
                      layer_us_after_write_only_flush=round(dirty2 * 1e3, 2)),
        "graph_replay": {"layer_us": round(graph_us, 2),
                         "value": round(wl2.T / (graph_us * 1e-6), 1), "unit": "tokens/s"},
        "e2e": {"value": round(wl2.T / (e2e2 * 1e-3), 1), "unit": "tokens/s",
                "ms_per_step": round(e2e2, 4), "h2d_bytes_per_step": h2d2,
                "d2h_bytes_per_step": d2h2, "in_flight": 3},
        "gpu_launches": run2.launches_per_step * n,
        "clocks": clk2.summary()})
    return out


def ffn_trace_run(run):
    """One more pass of the breakdown's step calls with the expert FFN's per-CTA
    record switched on (moe_set_ffn_trace): how the launch's tiles spread over
    the SMs.  Returns the tail summary of that launch."""
    torch, moe = run.torch, run.moe
    buf = torch.zeros((1024, 3), dtype=torch.int64, device=run.dev)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(run.part_names) + 1)]
    run.flush()
    moe.set_ffn_trace(buf)
    try:
        run.step_parts(evs)
        torch.cuda.synchronize()
    finally:
        moe.set_ffn_trace(None)
    tr = buf.cpu().numpy()
    tr = tr[tr[:, 1] > 0]
    return ffn_tail(tr)


def ffn_tail(tr):
    """Tail of one persistent FFN launch from its per-CTA record (rows: start ns,
    end ns, tiles).  idle_sm_frac: the share of CTA-time between the first
    CTA's start and the last CTA's end that CTAs spent not yet started or
    already finished; tail_us: from the first CTA to run out of tiles to the
    last one."""
    start, end, tiles = tr[:, 0].astype(np.float64), tr[:, 1].astype(np.float64), tr[:, 2]
    k0, k1 = start.min(), end.max()
    span = k1 - k0
    busy = end - start
    return {"ctas": int(len(tr)), "span_us": round(span / 1e3, 2),
            "idle_sm_frac": round(float(1.0 - busy.sum() / (len(tr) * span)), 4),
            "tail_us": round((k1 - end.min()) / 1e3, 2),
            "start_spread_us": round((start.max() - k0) / 1e3, 2),
            "end_p50_us": round((float(np.median(end)) - k0) / 1e3, 2),
            "tiles_per_cta": {"min": int(tiles.min()), "median": float(np.median(tiles)),
                              "max": int(tiles.max())}}


def skewed_line(dev, packed, steps, warmup, peaks, barrier):
    """The chunked prefill with 16 hot experts (+2.0 on their logits): whole-layer
    steps, the per-expert row counts, and the expert FFN against both roofs
    (at a mean of 128 rows per expert it sits below the ridge, so HBM and the
    tensor cores are both reported) with the tail of its grouped GEMM."""
    wl = synth.WORKLOADS["prefill_T2048_skewed"]
    run = LayerRun(wl, dev, packed)
    clk = ClockSampler(int(dev.index or 0))
    n = max(steps, 30)
    with clk:
        st, _ = run.timed(n, warmup, barrier)
    per = run.breakdown(n)
    tail = ffn_trace_run(run)
    counts = run.counts.cpu().numpy()
    T = wl.T
    ffn_ms = float(per[:, run.part_names.index("expert_ffn")].mean())
    d = int((counts > 0).sum())
    nbytes = d * (GATE_UP_BYTES_PER_EXPERT + DOWN_BYTES_PER_EXPERT) + T * 1536 * 2 + \
        8 * T * 1536 * 2
    flops = FLOPS_PER_ROW * 8 * T
    ms = float(st.mean())
    hot = set(int(e) for e in run.tok.hot_experts)
    return {"value": round(T / (ms * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 5),
            "T": T, "hot_experts": sorted(hot),
            "counts": [int(c) for c in counts],
            "M": {"max": int(counts.max()), "mean": round(float(counts.mean()), 2),
                  "max_over_mean": round(float(counts.max() / counts.mean()), 3),
                  "mean_hot": round(float(np.mean([counts[e] for e in hot])), 1),
                  "mean_other": round(float(np.mean([c for e, c in enumerate(counts)
                                                     if e not in hot])), 1)},
            "expert_ffn": {"us": round(ffn_ms * 1e3, 2), "distinct_experts": d,
                           "hbm_frac": round(nbytes / (ffn_ms * 1e-3) / 1e9 /
                                             float(peaks["hbm_gbs"]), 4),
                           "tensor_frac": round(flops / (ffn_ms * 1e-3) / 1e12 /
                                                float(peaks["bf16_tflops"]), 4),
                           "tail": tail},
            "layer": layer_fractions(wl, run, st, per, peaks),
            "gpu_launches": run.launches_per_step * n + len(run.part_names),
            "clocks": clk.summary()}


def decode_T4_line(dev, packed, steps, warmup, peaks, peak_kind, barrier):
    """Four concurrent decode streams, seeds 1..8, each seed its own batch:
    per-seed whole-layer time and the expert FFN's HBM fraction, and their
    medians."""
    per_seed = []
    launches = 0
    clk = ClockSampler(int(dev.index or 0))
    with clk:
        for s in range(1, 9):
            wl = synth.WORKLOADS[f"decode_T4_seed{s}"]
            run = LayerRun(wl, dev, packed)
            n = max(steps, 30)
            st, _ = run.timed(n, warmup, barrier)
            per = run.breakdown(n)
            rf = roofline_for(wl, run, per, peaks, peak_kind)
            lf = layer_fractions(wl, run, st, per, peaks)
            per_seed.append({"seed": s, "layer_us": lf["layer_us"],
                             "ffn_us": lf["kernel_us"]["expert_ffn"],
                             "distinct_experts": rf["distinct_experts"],
                             "ffn_hbm_frac": rf["frac"], "layer_hbm_frac": lf["hbm_frac"]})
            launches += run.launches_per_step * n
            del run
    med = {k: round(float(np.median([p[k] for p in per_seed])), 4)
           for k in ("layer_us", "ffn_us", "distinct_experts", "ffn_hbm_frac", "layer_hbm_frac")}
    return {"value": round(4 / (med["layer_us"] * 1e-6), 1), "unit": "tokens/s",
            "T": 4, "median": med, "per_seed": per_seed, "gpu_launches": launches,
            "clocks": clk.summary()}


def summary_of(line, main_name):
    """A short digest of every configuration's headline numbers, placed last on
    the JSON line so that the end of the output shows it."""
    bound = line["roofline"]["bound"]
    key = "tensor" if bound == "tensor" else "hbm"
    out = {main_name: {"us": line["layer"]["layer_us"],
                       f"ffn_{key}_frac": line["roofline"]["frac"],
                       f"layer_{key}_frac": line["layer"][f"{key}_frac"]}}
    if "decode_T16" in line:
        d = line["decode_T16"]
        out["decode_T16"] = {"us": d["layer"]["layer_us"], "ffn_hbm_frac": d["roofline"]["frac"],
                             "layer_hbm_frac": d["layer"]["hbm_frac"]}
    for k in ("decode_T16_fp8", "decode_T16_nvfp4"):
        if k in line:
            out[k] = {"us": line[k]["layer"]["layer_us"],
                      "ffn_hbm_frac": line[k]["roofline"]["frac"]}
    if "decode_T4" in line:
        m = line["decode_T4"]["median"]
        out["decode_T4_median"] = {"us": m["layer_us"], "ffn_hbm_frac": m["ffn_hbm_frac"]}
    if "prefill_T2048_skewed" in line:
        k = line["prefill_T2048_skewed"]
        out["prefill_T2048_skewed"] = {
            "us": round(k["ms_per_step"] * 1e3, 2), "max_over_mean_M": k["M"]["max_over_mean"],
            "ffn_hbm_frac": k["expert_ffn"]["hbm_frac"],
            "ffn_tensor_frac": k["expert_ffn"]["tensor_frac"],
            "ffn_idle_sm_frac": k["expert_ffn"]["tail"]["idle_sm_frac"]}
    for k in ("stack23_T1", "stack23_T8189", "stack23_T1_routed", "stack23_T8189_routed"):
        if k in line:
            out[k] = {"us_per_layer": line[k]["us_per_layer"], "tok_s": line[k]["value"]}
    for k in ("decode_T16_e256", "decode_T16_shared1"):
        if k in line:
            out[k] = {"us": round(line[k]["ms_per_step"] * 1e3, 2)}
    return out


def shared_layer(dev, n_shared):
    """n_shared synthetic shared experts of layer 0, packed."""
    import torch
    from group_limited_routed_moe_b200 import moe
    bits = synth.shared_weights_np(0, 0, n_shared)
    dev_t = [torch.from_numpy(b.view(np.int16)).to(dev).view(torch.bfloat16) for b in bits]
    return moe.moe_pack_shared(*dev_t), n_shared


def shared_line(wl2, dev, packed, shared, routed_ms, steps, warmup, peaks, barrier):
    """The decode batch with shared experts: whole-layer steps, and the shared
    experts' extra time against the routed-only layer, over their HBM bytes."""
    run = LayerRun(wl2, dev, packed, shared=shared)
    clk = ClockSampler(int(dev.index or 0))
    n = max(steps, 50)
    with clk:
        st, _ = run.timed(n, warmup, barrier)
    ms = float(st.mean())
    extra_us = (ms - routed_ms) * 1e3
    nbytes = shared[1] * (GATE_UP_BYTES_PER_EXPERT + DOWN_BYTES_PER_EXPERT) + \
        wl2.T * 1536 * 2 + shared[1] * wl2.T * 1536 * 2
    peak = float(peaks["hbm_gbs"])
    return {"value": round(wl2.T / (ms * 1e-3), 1), "unit": "tokens/s",
            "ms_per_step": round(ms, 5), "n_shared": shared[1],
            "shared_extra_us": round(extra_us, 2),
            "shared_roofline": {"bound": "hbm", "bytes": nbytes,
                                "achieved": round(nbytes / max(extra_us, 1e-3) / 1e3, 1),
                                "peak": peak, "unit": "GB/s",
                                "note": "the shared experts' weights, x and their y rows over the "
                                        "layer's extra time against the routed-only layer"},
            "gpu_launches": run.launches_per_step * n, "clocks": clk.summary()}


def e256_line(T, dev, steps, warmup, peaks, barrier, seed=5):
    """The second MoE shape (256 experts in 8 groups of 32, keep 4, top-6, plus
    2 shared experts) on T synthetic tokens: whole-layer steps through
    moe_layer_e256 after the same L2 flush, and the layer's fractions of the
    HBM and tensor roofs (the touched experts' weights and the layer's flops)."""
    import torch
    from group_limited_routed_moe_b200 import moe
    halves = []
    for half in (0, 1):
        w = [synth.e256_weight_bits_torch(0, 0, m, half, dev)
             for m in (synth.W_GATE, synth.W_UP, synth.W_DOWN)]
        halves.append(moe.moe_pack_weights(*w))
        del w
    sh_packed, n_sh = shared_layer(dev, 2)
    tok = synth.make_tokens_e256(T, seed)
    x = torch.from_numpy(tok.x_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    lg = torch.from_numpy(tok.logits).to(dev)
    bias = torch.from_numpy(tok.bias).to(dev)
    out = torch.empty((T, 1536), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((T, 6), dtype=torch.int32, device=dev)
    n = moe.layer_e256_workspace_bytes(T, n_sh)
    raw = torch.empty(n + 1024, dtype=torch.uint8, device=dev)
    ws = raw[(-raw.data_ptr()) % 1024:][:n]
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        moe.moe_layer_e256(x, lg, bias, halves[0], halves[1], sh_packed, n_sh, out=out,
                           topk_idx_out=idx, workspace=ws, stream=stream)

    def flush():
        flush_w.fill_(1)
        flush_r.max()
        torch.cuda._sleep(1_000_000)
    for _ in range(warmup):
        flush()
        step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    clk = ClockSampler(int(dev.index or 0))
    barrier()
    torch.cuda.synchronize()
    with clk:
        for k in range(steps):
            flush()
            evs[k][0].record(stream)
            step()
            evs[k][1].record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    d = int(np.unique(idx.cpu().numpy()).size)
    nbytes = (d + n_sh) * (GATE_UP_BYTES_PER_EXPERT + DOWN_BYTES_PER_EXPERT) + T * (1536 * 4 + 512)
    flops = FLOPS_PER_ROW * (6 + n_sh) * T
    nb = (T + 127) // 128
    launches = 4 + 2 + (2 if n_sh else 0) + 1  # route, count, scan, scatter; 2 FFN; shared; combine
    return {"value": round(T / (ms * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 5),
            "shape": "256 experts in 8 groups of 32, keep 4, top-6, 2 shared experts",
            "T": T, "distinct_experts": d, "count_sort_blocks": nb,
            "hbm_frac": round(nbytes / (ms * 1e-3) / 1e9 / float(peaks["hbm_gbs"]), 4),
            "tensor_frac": round(flops / (ms * 1e-3) / 1e12 / float(peaks["bf16_tflops"]), 4),
            "gpu_launches": launches * steps, "clocks": clk.summary()}


STACK_LAYERS, STACK_SEED = 23, 4


def stack_packs(dev):
    """The stack's 23 layers of independent bf16 experts (seed 4, layers 0..22),
    packed: 13.9 GB."""
    import torch
    from group_limited_routed_moe_b200 import moe
    packs = []
    for l in range(STACK_LAYERS):
        w = [synth.weight_bits_torch(STACK_SEED, l, m, dev)
             for m in (synth.W_GATE, synth.W_UP, synth.W_DOWN)]
        packs.append(moe.moe_pack_weights(*w))
        del w
    torch.cuda.synchronize()
    return packs


def stack_routers(dev):
    """The stack's 23 router matrices (seed 4, layers 0..22), packed."""
    import torch
    from group_limited_routed_moe_b200 import moe
    out = []
    for l in range(STACK_LAYERS):
        bits = synth.router_weight_bits_np(STACK_SEED, l)
        out.append(moe.moe_pack_router(
            torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)))
    return out


def stack_line(T, dev, packs, steps, warmup, peaks, barrier, routers=None):
    """The 23-layer stack on T tokens: seeded router logits per layer, a bf16
    residual add between layers, the 23 moe_layer calls captured once as a CUDA
    graph and replayed (no host sync between layers).  Each replay streams every
    layer's touched experts, far more than L2 holds, so there is no flush; the
    input is restored before each replay, outside the timed events.  With
    `routers`, every layer is moe_layer_routed: its logits are projected from
    its own input h by its own router matrix (activation-dependent routing),
    and the seeded logits are not used."""
    import torch
    from group_limited_routed_moe_b200 import moe
    tok = synth.make_tokens(T, STACK_SEED)
    x0 = torch.from_numpy(tok.x_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    h = x0.clone()
    lgs, bs = [], []
    for l in range(STACK_LAYERS):
        lg, b = synth.layer_logits(T, STACK_SEED, l)
        lgs.append(torch.from_numpy(lg).to(dev))
        bs.append(torch.from_numpy(b).to(dev))
    idx = [torch.empty((T, 8), dtype=torch.int32, device=dev) for _ in range(STACK_LAYERS)]
    ws = moe.alloc_layer_workspace(T, dev)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for l in range(STACK_LAYERS):
                if routers is None:
                    moe.moe_layer(h, lgs[l], bs[l], packs[l], residual=h, out=h,
                                  topk_idx_out=idx[l], workspace=ws, stream=s)
                else:
                    moe.moe_layer_routed(h, routers[l], bs[l], packs[l], residual=h, out=h,
                                         topk_idx_out=idx[l], workspace=ws, stream=s)
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    for _ in range(warmup):
        h.copy_(x0)
        g.replay()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    clk = ClockSampler(int(dev.index or 0))
    barrier()
    torch.cuda.synchronize()
    with clk:
        for a, b in evs:
            h.copy_(x0)
            a.record(cur)
            g.replay()
            b.record(cur)
        torch.cuda.synchronize()
    barrier()
    status = moe.get_device_status(int(dev.index or 0))
    del g
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    distinct = sum(int(torch.unique(i).numel()) for i in idx)
    nbytes = distinct * (GATE_UP_BYTES_PER_EXPERT + DOWN_BYTES_PER_EXPERT) + \
        STACK_LAYERS * T * (1536 * 4 + 512)
    flops = STACK_LAYERS * FLOPS_PER_ROW * 8 * T
    nb = (T + 127) // 128
    n_rp = 1 if T <= 64 else 2 if T <= 1024 else (3 if nb <= 256 else 4)
    if routers is not None:
        nbytes += STACK_LAYERS * 1536 * 128 * 2  # the router matrices
        flops += STACK_LAYERS * 2 * T * 1536 * 128
        if T > 64:
            n_rp += 1  # the tensor-core projection runs as its own launch above 64 tokens
    return {"value": round(T / (ms * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 4),
            "routing": ("from each layer's own input (moe_layer_routed: router projection, "
                        "routing and sort in one launch up to 8 tokens)" if routers is not None
                        else "seeded per-layer logits (moe_layer)"),
            "layers": STACK_LAYERS, "T": T, "us_per_layer": round(ms * 1e3 / STACK_LAYERS, 2),
            "distinct_experts_all_layers": distinct,
            "hbm_frac": round(nbytes / (ms * 1e-3) / 1e9 / float(peaks["hbm_gbs"]), 4),
            "tensor_frac": round(flops / (ms * 1e-3) / 1e12 / float(peaks["bf16_tflops"]), 4),
            "note": ("one CUDA graph of 23 moe_layer calls per step (bf16 residual add fused into "
                     "the combine), no host sync between layers; no L2 flush (each step streams "
                     f"{nbytes / 1e9:.2f} GB of expert weights)"),
            "status_ok": status == moe.MOE_OK,
            "gpu_launches": (n_rp + (1 if T <= FUSED_COMBINE_MAX_T else 2)) * STACK_LAYERS * steps,
            "clocks": clk.summary()}


def fp8_layer(dev):
    """The synthetic block-FP8 checkpoint of layer 0 (power-of-two block scales),
    packed, and its host codes and scales."""
    from group_limited_routed_moe_b200 import moe
    qs = []
    for which in (synth.W_GATE, synth.W_UP, synth.W_DOWN):
        q, sc = synth.fp8_weights_torch(0, 0, which, dev, "pow2")
        qs += [q, sc]
    packed = moe.moe_pack_weights_fp8(*qs)
    return packed, qs


def nvfp4_layer(dev):
    """The synthetic NVFP4 checkpoint of layer 0 (power-of-two tensor scales),
    packed, and its codes and scales on the device."""
    from group_limited_routed_moe_b200 import moe
    qs = []
    for which in (synth.W_GATE, synth.W_UP, synth.W_DOWN):
        qs += list(synth.nvfp4_weights_torch(0, 0, which, dev, "pow2"))
    packed = moe.moe_pack_weights_nvfp4(*qs)
    return packed, qs


def run_ours(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if dist is not None:
            dist.barrier()

    from group_limited_routed_moe_b200 import moe
    peaks, peak_kind = load_peaks()

    wg = synth.weight_bits_torch(0, 0, synth.W_GATE, dev)
    wu = synth.weight_bits_torch(0, 0, synth.W_UP, dev)
    wd = synth.weight_bits_torch(0, 0, synth.W_DOWN, dev)
    packed = moe.moe_pack_weights(wg, wu, wd)
    torch.cuda.synchronize()

    def host_weights():
        def h(t):
            return t.view(torch.int16).cpu().numpy().view(np.uint16)
        return h(wg), h(wu), h(wd)

    fp8_packed, fp8_dev = fp8_layer(dev) if (args.weights == "fp8" or not args.no_secondary) \
        else (None, None)
    fp4_packed, fp4_dev = nvfp4_layer(dev) if (args.weights == "nvfp4" or not args.no_secondary) \
        else (None, None)
    torch.cuda.synchronize()
    fp8 = args.weights == "fp8"
    nvfp4 = args.weights == "nvfp4"
    wl = synth.WORKLOADS[args.workload]
    shared = shared_layer(dev, args.shared) if args.shared > 0 else None
    main_w = fp4_packed if nvfp4 else fp8_packed if fp8 else packed
    run = LayerRun(wl, dev, main_w, fp8=fp8, shared=shared, nvfp4=nvfp4)
    clk = ClockSampler(local)
    with clk:
        steps_ms, wall = run.timed(args.steps, args.warmup, barrier)
    per = run.breakdown(args.steps)
    dirty_ms = run.dirty_l2_steps(args.steps, barrier)
    router = run.router(max(10, args.steps // 5), peaks)
    step_ms = float(steps_ms.mean())
    ms_per_step = max_over_ranks(step_ms * args.steps, dist, dev) / args.steps
    value = job_tokens_per_s(wl.T, world, ms_per_step)
    e2e_ms, h2d, d2h = run.e2e(max(8, args.steps // 2), 3)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)

    line = {
        "metric": f"MoE-layer tokens/s ({wl.name}: T={wl.T}, hidden 1536, 128 experts top-8)",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "T_buf": wl.T_buf, "hidden": 1536,
                   "weights": ("block-FP8 experts (E4M3 codes, power-of-two 128x128 block scales)"
                               if fp8 else
                               "NVFP4 experts (E2M1 codes, E4M3 scales per 16, power-of-two "
                               "tensor scales)" if nvfp4 else "bf16 experts"),
                   "shared_experts": args.shared,
                   "experts": 128, "groups": 8, "keep_groups": 4, "topk": 8, "inter": 512,
                   "parallelism": f"dp{world} (independent batch per GPU)",
                   "l2": ("256 MB buffer overwritten, then another 256 MB buffer read, before "
                          "every step (outside the timed events): no line of the inputs and no "
                          "dirty line is left in L2"),
                   "wall_s_timed_region": round(wall, 4)},
        "roofline": roofline_for(wl, run, per, peaks, peak_kind),
        "router": router,
        "layer": dict(layer_fractions(wl, run, steps_ms, per, peaks),
                      layer_us_after_write_only_flush=round(dirty_ms * 1e3, 2),
                      ffn_tail=ffn_trace_run(run)),
        "e2e": {"value": round(job_tokens_per_s(wl.T, world, e2e_ms), 1), "unit": "tokens/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "in_flight": 3,
                "note": ("moe.HostPipeline over the C ABI's moe_layer_host: each step copies "
                         "its inputs in and its output out (one cudaMemcpyAsync per buffer); "
                         "3 steps in flight on 3 streams, their copies overlapping the "
                         "other step's layer, the layers one after another; no L2 flush "
                         "(each step streams the touched experts' weights, more than L2 holds)")},
        "gpu_launches": run.launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if not args.no_secondary:
        wl2 = synth.WORKLOADS["decode_T16"]
        for key, p2, fmt in (("decode_T16", packed, "bf16"), ("decode_T16_fp8", fp8_packed, "fp8"),
                             ("decode_T16_nvfp4", fp4_packed, "nvfp4")):
            if wl2.name == wl.name and fmt == args.weights:
                continue  # that is the main line
            line[key] = decode_line(wl2, dev, p2, fmt == "fp8", args.steps, args.warmup, peaks,
                                    peak_kind, barrier, nvfp4=fmt == "nvfp4")
            line["gpu_launches"] += line[key]["gpu_launches"]
        line["decode_T16_e256"] = e256_line(16, dev, max(args.steps, 50), args.warmup, peaks,
                                            barrier)
        line["gpu_launches"] += line["decode_T16_e256"]["gpu_launches"]
        if "decode_T16" in line:
            key = "decode_T16_shared1"
            line[key] = shared_line(wl2, dev, packed, shared_layer(dev, 1),
                                    line["decode_T16"]["ms_per_step"], args.steps, args.warmup,
                                    peaks, barrier)
            line["gpu_launches"] += line[key]["gpu_launches"]
    if not args.no_configs:
        line["decode_T4"] = decode_T4_line(dev, packed, args.steps, args.warmup, peaks, peak_kind,
                                           barrier)
        line["gpu_launches"] += line["decode_T4"]["gpu_launches"]
        line["prefill_T2048_skewed"] = skewed_line(dev, packed, args.steps, args.warmup, peaks,
                                                   barrier)
        line["gpu_launches"] += line["prefill_T2048_skewed"]["gpu_launches"]
    if not args.no_stack:
        packs = stack_packs(dev)
        routers = stack_routers(dev)
        # both decode stacks first: right after a prefill stack the SM clock was
        # seen settling below its maximum for a while
        for T_s, key, rt in ((1, "stack23_T1", None), (1, "stack23_T1_routed", routers),
                             (8189, "stack23_T8189", None),
                             (8189, "stack23_T8189_routed", routers)):
            n = max(10, args.steps // 2) if T_s == 1 else max(5, args.steps // 10)
            line[key] = stack_line(T_s, dev, packs, n, args.warmup, peaks, barrier, routers=rt)
            line["gpu_launches"] += line[key]["gpu_launches"]
        del packs
    if args.e256_prefill:
        line["prefill_T8189_e256"] = e256_line(8189, dev, max(5, args.steps // 5), args.warmup,
                                               peaks, barrier)
        line["gpu_launches"] += line["prefill_T8189_e256"]["gpu_launches"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if fp8 or nvfp4:
            hw = [t.cpu().numpy() for t in (fp4_dev if nvfp4 else fp8_dev)]
        else:
            hw = host_weights()
        line["cpu_baseline"] = cpu_baseline(wl, run.tok, hw, args.cpu_sample, fp8=fp8,
                                            nvfp4=nvfp4)
    line["summary"] = summary_of(line, wl.name)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The float64 oracle as the reference arm: rank 0 only, host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle as O
    from threadpoolctl import threadpool_info
    wl = synth.WORKLOADS[args.workload]
    tok = synth.make_tokens(wl.T, wl.seed, hot=wl.hot)
    per_step = min(wl.T, 64)
    rr = O.route(tok.logits, tok.bias)
    host_w = synth.layer_weights_np(0, 0)
    for k in range(args.warmup):
        rows = (np.arange(per_step) + k * per_step) % wl.T
        O.moe_layer(tok.x_bits[rows], tok.logits[rows], tok.bias, *host_w)
    t0 = time.perf_counter()
    for k in range(args.steps):
        rows = (np.arange(per_step) + k * per_step) % wl.T
        O.moe_layer(tok.x_bits[rows], tok.logits[rows], tok.bias, *host_w)
    dt = time.perf_counter() - t0
    del rr
    value = per_step * args.steps / dt
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    line = {
        "impl": "reference",
        "metric": f"MoE-layer tokens/s ({wl.name}: T={wl.T}, hidden 1536, 128 experts top-8)",
        "value": round(value, 2), "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "T_buf": wl.T_buf,
                   "step": f"{per_step} tokens of the batch per step"},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": threads,
                         "kind": "oracle",
                         "sample": f"{per_step} tokens per step x {args.steps} steps of {wl.name}"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
