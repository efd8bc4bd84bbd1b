"""Throughput of the kernelized linear attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--case NAME] [--no-configs] [--no-cpu-baseline]

One run measures every workload of the pages (kernelized_linear_attention_phi_b200/
workloads.py) and prints ONE JSON line. Its headline (``value``, ``e2e``,
``roofline``, ``cpu_baseline``) is the largest workload that one GPU holds,
the long-context case: a step is one non-causal call on B=4, H=16, N=16384
(128x128 latent tokens), d=64 plus one causal call on B=1, H=16, N=131072,
d=128, both bf16, phi = relu+1, normalized. ``per_config`` holds the same
fields for every other workload:

* ``single_head``: 1x1x256x16 fp32, non-causal;
* ``multi_head_bf16`` / ``multi_head_f32``: 2x8x4096x64, non-causal + causal
  (chunk 64);
* ``prefix_mask``: 8x8x2048x64 bf16, identity map, unnormalized, m_i uniform
  in [0, N-1]; ``prefix_mask_arange``: the same with m = arange(N);
* ``decode``: 64 sequences x 32 heads, d=128, fp32 state prefilled from 2048
  bf16 tokens; a step is 1024 one-token decode steps;
* ``multi_head_bwd_bf16``: the gradients (dq, dk, dv) of both 2x8x4096x64
  forms.

Tokens per step: B*N per full-sequence call, sequences x steps for decode.
``value`` is tokens/s over all ranks (weak scaling: each rank runs its own
batch; the path has no exchange step, so there is no data-path collective).
Each library call is captured once into a CUDA graph (decode: the 1024
steps in one graph) and the graphs are replayed. Timing: CUDA events around
every call on the launching stream, L2 flushed (a 256 MiB write) before
every call outside the events, W untimed warm-up steps, max over ranks.
``e2e`` repeats the step through the plain API calls with pinned host inputs
copied in and the outputs copied back inside the timed region, the copies of
one step overlapped with the calls of the previous (separate copy streams,
double-buffered device tensors) or run back to back on one stream
(``e2e.serial_value``), whichever is faster (``e2e.schedule``).
``roofline`` is the dominant kernel's: after the timed steps every call is
replayed from a graph captured with the library's per-kernel timing events
(la_timing_enable), L2 flushed before each replay, and the kernel with the
largest mean time has its algorithmic bytes divided by that time (decode:
the 1024-step call time over 1024).
"""

from __future__ import annotations

import argparse
import datetime
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

from kernelized_linear_attention_phi_b200 import workloads as W  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
METRIC = "tokens/sec (fwd, 1xB200) and % of HBM / bf16 tensor-core roofline per kernel"

# The calls of each case: (workload, dtype, form, mask kind).
CASES = {
    "long": [("long_noncausal", "bf16", "noncausal", None), ("long_causal", "bf16", "causal", None)],
    "single_head": [("single_head", "f32", "noncausal", None)],
    "multi_head_bf16": [("multi_head", "bf16", "noncausal", None), ("multi_head", "bf16", "causal", None)],
    "multi_head_f32": [("multi_head", "f32", "noncausal", None), ("multi_head", "f32", "causal", None)],
    "prefix_mask": [("prefix_mask", "bf16", "prefix", "uniform")],
    "prefix_mask_arange": [("prefix_mask", "bf16", "prefix", "arange")],
    "decode": [("decode", "bf16", "decode", None)],
    "multi_head_bwd_bf16": [("multi_head_bwd", "bf16", "noncausal_bwd", None),
                            ("multi_head_bwd", "bf16", "causal_bwd", None)],
}
HEADLINE = "long"
CASE_TEXT = {
    "long": "long-context: non-causal 4x16x16384x64 (128x128 latent tokens) + causal 1x16x131072x128, bf16, "
            "phi=relu1, normalized",
    "single_head": "single head: non-causal 1x1x256x16 fp32, phi=relu1, normalized",
    "multi_head_bf16": "multi-head: non-causal + causal (chunk 64) 2x8x4096x64 bf16, phi=relu1, normalized",
    "multi_head_f32": "multi-head: non-causal + causal (chunk 64) 2x8x4096x64 fp32, phi=relu1, normalized",
    "prefix_mask": "prefix mask: 8x8x2048x64 bf16, identity map, unnormalized, m_i uniform in [0, N-1]",
    "prefix_mask_arange": "prefix mask: 8x8x2048x64 bf16, identity map, unnormalized, m = arange(N)",
    "decode": "decode: 64 sequences x 32 heads, d=128, fp32 state prefilled from 2048 bf16 tokens, "
              "1024 one-token steps per step",
    "multi_head_bwd_bf16": "gradients: dq, dk, dv of non-causal + causal 2x8x4096x64 bf16, upstream N(0,1)",
}

# Kernels each call launches, in launch order, by the number the library's
# timing events report (the dispatch in la_api.cu takes one-launch or
# in-cluster-scan paths where the problem allows; the count tells which).
TC_KERNELS = {
    "noncausal": {1: ["tc_noncausal_cluster_kernel"],
                  3: ["tc_kv_kernel", "kv_reduce_balanced_kernel", "tc_readout_kernel"]},
    "causal": {2: ["tc_kv_kernel", "tc_sweep"], 3: ["tc_kv_kernel", "state_scan_kernel", "tc_sweep"]},
    "prefix": {3: ["tc_kv_kernel", "bin_kernel", "tc_sweep"],
               4: ["tc_kv_kernel", "bin_kernel", "state_scan_kernel", "tc_sweep"]},
    "decode": {1: ["decode_kernel"]},
    "noncausal_bwd": {4: ["tc_noncausal_cluster_kernel", "tc_bwd_q_kernel", "kv_reduce_balanced_kernel",
                          "tc_bwd_kv_kernel"],
                      5: ["tc_kv_kernel", "kv_reduce_balanced_kernel", "tc_bwd_q_kernel",
                          "kv_reduce_balanced_kernel", "tc_bwd_kv_kernel"]},
    "causal_bwd": {4: ["tc_kv_kernel", "tc_bwd_causal_q_kernel", "state_scan_kernel", "tc_bwd_causal_kv_kernel"],
                   5: ["tc_kv_kernel", "state_scan_kernel", "tc_bwd_causal_q_kernel", "state_scan_kernel",
                       "tc_bwd_causal_kv_kernel"]},
}
SIMT_KERNELS = {
    "noncausal": {1: ["noncausal_small_kernel"], 3: ["kv_partial_kernel", "state_reduce_kernel", "readout_kernel"]},
    "causal": {3: ["kv_partial_kernel", "state_scan_kernel", "chunked_kernel"]},
    "prefix": {4: ["kv_partial_kernel", "bin_kernel", "state_scan_kernel", "chunked_kernel"]},
    "decode": {1: ["decode_kernel"]},
    "noncausal_bwd": {5: ["kv_partial_kernel", "state_reduce_kernel", "bwd_q_kernel", "state_reduce_kernel",
                          "bwd_kv_kernel"]},
    "causal_bwd": {5: ["kv_partial_kernel", "state_scan_kernel", "bwd_q_kernel", "state_scan_kernel",
                       "bwd_kv_kernel"]},
}
# fp32 at d = 64: the split-precision tensor-core kernel in its four modes
# (block / split states, causal sweep, readout, prefix-mask sweep); decode and
# the gradient sweeps stay on the CUDA cores
F32_TC_KERNELS = dict(SIMT_KERNELS)
F32_TC_KERNELS.update({
    "noncausal": {3: ["tc_f32_kernel<0", "state_reduce_kernel", "tc_f32_kernel<2"]},
    "causal": {3: ["tc_f32_kernel<0", "state_scan_kernel", "tc_f32_kernel<1"]},
    "prefix": {4: ["tc_f32_kernel<0", "bin_kernel", "state_scan_kernel", "tc_f32_kernel<3"]},
    "noncausal_bwd": {5: ["tc_f32_kernel<0", "state_reduce_kernel", "bwd_q_kernel", "state_reduce_kernel",
                          "bwd_kv_kernel"]},
    "causal_bwd": {5: ["tc_f32_kernel<0", "state_scan_kernel", "bwd_q_kernel", "state_scan_kernel",
                       "bwd_kv_kernel"]},
})

# What each kernel does, for its algorithmic bytes (Call.kernel_bytes).
KERNEL_ROLE = {"tc_kv_kernel": "kv", "kv_partial_kernel": "kv", "kv_reduce_balanced_kernel": "reduce",
               "state_reduce_kernel": "reduce", "tc_readout_kernel": "readout", "readout_kernel": "readout",
               "state_scan_kernel": "scan", "tc_sweep": "sweep", "chunked_kernel": "sweep",
               "bin_kernel": "bin", "decode_kernel": "decode", "bwd_q_kernel": "bwd_q",
               "bwd_kv_kernel": "bwd_kv", "tc_bwd_q_kernel": "bwd_q", "tc_bwd_kv_kernel": "bwd_kv",
               "tc_bwd_causal_q_kernel": "bwd_q", "tc_bwd_causal_kv_kernel": "bwd_kv",
               "tc_noncausal_cluster_kernel": "fused", "noncausal_small_kernel": "fused", "tc_f32_kernel<0": "kv", "tc_f32_kernel<1": "sweep",
               "tc_f32_kernel<2": "readout", "tc_f32_kernel<3": "sweep"}


def block_plan(B, H, N, d, dtype, sms):
    """(block_tokens, nblk) of the chunked forms, as the library plans them
    (csrc/plan.h block_plan): one wave of CTAs (one per SM for d = 128, else
    two), blocks of at least 256 tokens in multiples of 128."""
    per_sm = 1 if d == 128 else 2
    target = max(1, per_sm * sms // (B * H))
    bt = max(256, -(-(-(-N // target)) // 128) * 128)
    return bt, -(-N // bt)


def kernel_table(dtype, d):
    """The kernels the library runs a problem on: tensor cores for bf16 with
    d = 64 or 128 and (split precision) fp32 with d = 64; CUDA cores otherwise."""
    if dtype == "bf16" and d in (64, 128):
        return TC_KERNELS
    return F32_TC_KERNELS if dtype == "f32" and d == 64 else SIMT_KERNELS


def kernel_names(form, dtype, d, count):
    """Names of the `count` kernels a call of `form` launched."""
    names = kernel_table(dtype, d).get(form, {}).get(count)
    return names if names else [f"kernel{i}" for i in range(count)]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--case", default=HEADLINE, choices=sorted(CASES),
                    help="the case the headline fields measure (default: the long-context step)")
    ap.add_argument("--no-configs", action="store_true", help="measure the headline case only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--record-traffic", metavar="NCU_CSV",
                    help="read an ncu launch list with dram__bytes_read.sum and dram__bytes_write.sum "
                         "of a --case run (--no-configs) and store its calls' DRAM bytes in "
                         "profiles/traffic.json; --traffic-scale multiplies them (a capture of a "
                         "smaller problem scaled to the case's size)")
    ap.add_argument("--traffic-scale", type=float, default=1.0)
    ap.add_argument("--scale-heads", type=int, default=0,
                    help="run the case with this many heads instead of the workload's (for a "
                         "reduced-size ncu capture; never a bench number)")
    return ap.parse_args(argv)


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


# ---------------------------------------------------------------------------
# Clock sampling (NVML reads only; no setting is changed)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._active = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            pr = torch.cuda.get_device_properties(device)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _sample(self):
        self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        try:
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.reasons |= int(r) & ~0x1

    def _run(self):
        while not self._stop.is_set():
            if self._active.is_set():
                self._sample()
            time.sleep(0.01)

    def start(self):
        if self.nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def timed(self):
        """Context manager: sample while a timed region runs."""
        sampler = self

        class _Region:
            def __enter__(self):
                sampler._active.set()

            def __exit__(self, *a):
                if sampler.nv:
                    sampler._sample()
                sampler._active.clear()
        return _Region()

    def stop(self):
        if self.nv:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.nv or not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples),
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b]}


# ---------------------------------------------------------------------------
# One library call on its own seeded inputs
# ---------------------------------------------------------------------------

class Call:
    """Device buffers and the library call of one (workload, dtype, form)."""

    def __init__(self, wl, dtype, form, mask, seed, device, heads=0):
        from kernelized_linear_attention_phi_b200 import binding as la
        self.la, self.wl, self.dtype, self.form, self.mask = la, wl, dtype, form, mask
        B, H, N, d = wl.B, (heads or wl.H), wl.N, wl.d
        self.B, self.H, self.N, self.d = B, H, N, d
        self.name = wl.name if form != "prefix" or mask == "uniform" else f"{wl.name}_{mask}"
        self.phi, self.normalize, self.chunk = wl.phi, wl.normalize, wl.chunk
        self.seed = seed
        self.sms = torch.cuda.get_device_properties(device).multi_processor_count
        self.ws = None
        self.elem = 2 if dtype == "bf16" else 4
        desc = la.make_desc(B, H, N, d, W.TORCH_DTYPES[dtype], self.phi, self.normalize)
        if form == "decode":
            T = wl.decode_steps
            self.steps = T
            _, k0, v0 = W.qkv(B, H, N, d, wl.sigma, seed, dtype, device)
            self.S = torch.empty(B, H, d, d, dtype=torch.float32, device=device)
            self.z = torch.empty(B, H, d, dtype=torch.float32, device=device)
            la.la_kv_summary(k0, v0, self.S, self.z, self.phi)  # the cached state: a prefill of N tokens
            del k0, v0
            self.qs, self.ks, self.vs = W.decode_tokens(T, B, H, d, wl.sigma, seed + 1, dtype, device)
            self.outs = torch.empty_like(self.qs)
            self.tokens = B * T
        else:
            self.steps = 1
            self.q, self.k, self.v = W.qkv(B, H, N, d, wl.sigma, seed, dtype, device)
            if form == "prefix":
                self.m = (W.prefix_mask_uniform(B, N, seed, device) if mask == "uniform"
                          else W.prefix_mask_arange(B, N, device))
            if form.endswith("_bwd"):
                self.dout = W.upstream_grad(B, H, N, d, seed, dtype, device)
                self.grads = tuple(torch.empty_like(self.q) for _ in range(3))
            else:
                self.out = torch.empty_like(self.q)
            op = {"prefix": "prefix", "causal": "causal"}.get(form, form)
            self.ws = la.workspace(desc, op, self.chunk, device)
            self.tokens = B * N

    def run(self):
        la = self.la
        f = self.form
        if f == "noncausal":
            la.la_noncausal(self.q, self.k, self.v, self.out, None, None, self.phi, self.normalize, self.ws)
        elif f == "causal":
            la.la_causal_chunked(self.q, self.k, self.v, self.out, self.chunk, self.phi, self.normalize, self.ws)
        elif f == "prefix":
            la.la_prefix_mask(self.q, self.k, self.v, self.m, self.out, self.chunk, self.phi, self.normalize,
                              self.ws)
        elif f == "decode":
            for t in range(self.steps):
                la.la_decode_step(self.qs[t], self.ks[t], self.vs[t], self.S, self.z, self.outs[t], self.phi,
                                  self.normalize)
        elif f == "noncausal_bwd":
            la.la_noncausal_backward(self.q, self.k, self.v, self.dout, *self.grads, self.phi, self.normalize,
                                     self.ws)
        elif f == "causal_bwd":
            la.la_causal_backward(self.q, self.k, self.v, self.dout, *self.grads, self.phi, self.normalize, self.ws)

    def run_from_host(self, h_ins, h_outs):
        """The call through the public API with its inputs copied in from
        pinned host memory and its outputs copied back (decode: per step)."""
        if self.form == "decode":
            hq, hk, hv = h_ins
            (ho,) = h_outs
            for t in range(self.steps):
                self.qs[t].copy_(hq[t], non_blocking=True)
                self.ks[t].copy_(hk[t], non_blocking=True)
                self.vs[t].copy_(hv[t], non_blocking=True)
                self.la.la_decode_step(self.qs[t], self.ks[t], self.vs[t], self.S, self.z, self.outs[t], self.phi,
                                       self.normalize)
                ho[t].copy_(self.outs[t], non_blocking=True)
            return
        ins, outs = self.device_io()
        for d_t, h_t in zip(ins, h_ins):
            d_t.copy_(h_t, non_blocking=True)
        self.run()
        for h_t, d_t in zip(h_outs, outs):
            h_t.copy_(d_t, non_blocking=True)

    def device_io(self):
        if self.form == "decode":
            return [self.qs, self.ks, self.vs], [self.outs]
        ins = [self.q, self.k, self.v] + ([self.m] if self.form == "prefix" else []) \
            + ([self.dout] if self.form.endswith("_bwd") else [])
        outs = list(self.grads) if self.form.endswith("_bwd") else [self.out]
        return ins, outs

    def bind_io(self, ins, outs):
        """Point the call at other device tensors of the same shapes (the
        order of device_io)."""
        self.q, self.k, self.v = ins[:3]
        rest = ins[3:]
        if self.form == "prefix":
            self.m, rest = rest[0], rest[1:]
        if self.form.endswith("_bwd"):
            self.dout = rest[0]
            self.grads = tuple(outs)
        else:
            self.out = outs[0]

    def algorithmic_bytes(self):
        """Bytes the call must move at least: its inputs once and outputs once."""
        t = self.B * self.H * self.N * self.d * self.elem     # one [B,H,N,d] tensor
        st = self.B * self.H * (self.d * self.d + self.d) * 4  # fp32 (S, z)
        one = self.B * self.H * self.d * self.elem
        return {"noncausal": 4 * t, "causal": 4 * t, "prefix": 4 * t + self.B * self.N * 4,
                "decode": self.steps * (2 * st + 4 * one), "noncausal_bwd": 7 * t, "causal_bwd": 7 * t}[self.form]

    def kernel_bytes(self, kernel):
        """Algorithmic bytes of one kernel launch of the call: the method's
        tensors it must read or write once (Q, K, V, out, S, z, m). Scratch
        the library keeps between its kernels (partial and block-state
        records, the binning tables) is not counted, so a kernel that only
        moves scratch (the prefix scan over block states) has none."""
        kb = kernel_bytes(self.form, kernel, self.B, self.H, self.N, self.d, self.elem)
        if self.form == "causal" and self.dtype == "bf16" and self.d == 128 and KERNEL_ROLE.get(kernel) == "kv":
            # the d = 128 causal call forms the states of every block but the
            # last (no prefix holds it): the KV pass reads those keys only
            bt, nblk = block_plan(self.B, self.H, self.N, self.d, self.dtype, self.sms)
            if nblk >= 2:
                kb = kb * min(self.N, (nblk - 1) * bt) // self.N
        return kb


def e2e_pipelined(calls, h_io, steps, stream):
    """Seconds for `steps` steps through the public API with every step's
    inputs copied in from pinned host memory and its outputs copied back, the
    copies overlapped with the calls: host-to-device copies on one stream, the
    calls on `stream`, device-to-host copies on a third; each call's device
    tensors are double-buffered, and a buffer is refilled only after the call
    that read it, and emptied only after the copy that read it, are done.
    Timed on the device from before the first copy in to after the last copy
    out."""
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    bufs = []
    for c in calls:
        ins, outs = c.device_io()
        bufs.append(([ins, [torch.empty_like(t) for t in ins]], [outs, [torch.empty_like(t) for t in outs]]))
    ev = lambda: torch.cuda.Event()
    done, freed = {}, {}
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(s_in)
    for i in range(steps):
        for j, (c, (h_ins, h_outs)) in enumerate(zip(calls, h_io)):
            (ins, outs), b = bufs[j], i % 2
            if i >= 2:
                s_in.wait_event(done[j, i - 2])
            with torch.cuda.stream(s_in):
                for d_t, h_t in zip(ins[b], h_ins):
                    d_t.copy_(h_t, non_blocking=True)
            loaded = ev()
            loaded.record(s_in)
            stream.wait_event(loaded)
            if i >= 2:
                stream.wait_event(freed[j, i - 2])
            c.bind_io(ins[b], outs[b])
            with torch.cuda.stream(stream):
                c.run()
            done[j, i] = ev()
            done[j, i].record(stream)
            s_out.wait_event(done[j, i])
            with torch.cuda.stream(s_out):
                for h_t, d_t in zip(h_outs, outs[b]):
                    h_t.copy_(d_t, non_blocking=True)
            freed[j, i] = ev()
            freed[j, i].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize()
    for j, c in enumerate(calls):
        c.bind_io(*[x[0] for x in bufs[j]])
    return t0.elapsed_time(t1) / 1e3


def kernel_bytes(form, kernel, B, H, N, d, elem):
    t = B * H * N * d * elem
    st = B * H * (d * d + d) * 4
    one = B * H * d * elem
    role = KERNEL_ROLE.get(kernel)
    if form.endswith("_bwd"):
        # gradients: q, k, v, dout read and dq, dk, dv written once over
        # the sweeps (non-causal: q, dout -> dq; k, v -> dk, dv; causal:
        # q, k, v, dout -> dq; q, k, v -> dk, dv); the reductions of
        # (G, h) move scratch only
        causal = form == "causal_bwd"
        return {"kv": 2 * t, "fused": 2 * t, "bwd_q": (5 if causal else 3) * t,
                "bwd_kv": (5 if causal else 4) * t}.get(role, 0)
    return {"kv": 2 * t, "reduce": st, "readout": 2 * t + st, "scan": 0, "sweep": 4 * t, "fused": 4 * t,
            "bin": B * N * 4, "decode": 2 * st + 4 * one}.get(role, 0)


def flush_l2(buf):
    buf.add_(1)


def rank_seed(wl, rank):
    """Each rank runs its own batch (weak scaling): the workload's seed
    shifted by the rank."""
    return wl.seed + 1000 * rank


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate_tokens_per_s(tokens_per_step, steps, world, seconds):
    """Whole-job throughput: the tokens every rank processed over the slowest
    rank's time."""
    return tokens_per_step * steps * world / seconds


def e2e_choice(pipelined_s, serial_s, pipelinable):
    """The end-to-end figure is the faster of the two schedules of the same
    copies and calls (small steps: the serial one, whose single stream has no
    cross-stream event waits); decode steps have only the serial one.
    Returns (schedule, seconds)."""
    if pipelinable and pipelined_s < serial_s:
        return "pipelined", pipelined_s
    return "serial", serial_s


def kernel_times(call, flush, reps):
    """Mean duration (ms) of each kernel the call launches, from the
    library's timing events over `reps` replays of a graph of the call, L2
    flushed before each. Decode: the 1024-step call's time over 1024 (one
    kernel, back to back)."""
    la = call.la
    g = torch.cuda.CUDAGraph()
    if call.form == "decode":
        with torch.cuda.graph(g):
            call.run()
        g.replay()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            flush_l2(flush)
            a.record()
            g.replay()
            b.record()
        torch.cuda.synchronize()
        return [sum(a.elapsed_time(b) for a, b in ev) / reps / call.steps]
    la.la_timing_enable(True)
    try:
        with torch.cuda.graph(g):
            call.run()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        acc = None
        for _ in range(reps):
            flush_l2(flush)
            g.replay()
            ms = la.la_timing_read()
            acc = ms if acc is None else [a + b for a, b in zip(acc, ms)]
    finally:
        la.la_timing_enable(False)
    del g
    return [a / reps for a in acc]


def measure_case(case, args, rank, world, device, flush, sampler, peak, heads=0):
    """Times one case; returns its JSON fields (value, roofline, e2e, ...)."""
    calls = [Call(W.WORKLOADS[w], dt, form, mask, rank_seed(W.WORKLOADS[w], rank), device, heads)
             for w, dt, form, mask in CASES[case]]
    warm = max(args.warmup, 3)
    for _ in range(warm):
        for c in calls:
            c.run()
    torch.cuda.synchronize()
    graphs = []
    for c in calls:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            c.run()
        graphs.append(g)
    for _ in range(warm):
        for g in graphs:
            g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)

    K = args.steps
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # Every call starts with a cold L2 (a 256 MiB write before each call,
    # outside the events), so each reads its inputs from HBM; a step's time
    # is the sum of its calls' times.
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
          for _ in range(K)]
    with sampler.timed():
        for i in range(K):
            for j, g in enumerate(graphs):
                flush_l2(flush)
                ev[i][j][0].record(stream)
                g.replay()
                ev[i][j][1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    per_call_ms = [sum(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(K)) / K for j in range(len(calls))]
    del graphs

    # end to end through the public API: pinned host inputs in, outputs back
    h_io = []
    h2d = d2h = 0
    for c in calls:
        ins, outs = c.device_io()
        h_ins = [t.cpu().pin_memory() for t in ins]
        h_outs = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
        h2d += sum(t.numel() * t.element_size() for t in h_ins)
        d2h += sum(t.numel() * t.element_size() for t in h_outs)
        h_io.append((h_ins, h_outs))
    Ke = max(1, min(K, 20))
    # serial: each step's copies in, calls and copies out back to back on one stream
    e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Ke)]
    torch.cuda.synchronize()
    for i in range(Ke):
        flush_l2(flush)
        e_ev[i][0].record(stream)
        for c, (h_ins, h_outs) in zip(calls, h_io):
            c.run_from_host(h_ins, h_outs)
        e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_serial_s = sum(a.elapsed_time(b) for a, b in e_ev) / 1e3
    # pipelined: step i+1's copies in overlap step i's calls and copies out
    pipelinable = all(c.form != "decode" for c in calls)
    e2e_pipe_s = e2e_pipelined(calls, h_io, Ke, stream) if pipelinable else e2e_serial_s
    del h_io

    # each kernel's own duration (per-kernel timing events)
    kt = [kernel_times(c, flush, max(3, min(K, 20))) for c in calls]

    # every call reports expired bounded waits in its workspace error word
    bad_flags = {}
    for c in calls:
        if c.ws is not None:
            f = c.la.la_last_error(c.ws)[1]
            if f:
                bad_flags[f"{c.name}/{c.form}"] = f

    step_ms = sum(per_call_ms)
    t_s, e2e_pipe_s, e2e_serial_s = max_over_ranks([step_ms / 1e3 * K, e2e_pipe_s, e2e_serial_s], device)
    tokens = sum(c.tokens for c in calls)
    value = aggregate_tokens_per_s(tokens, K, world, t_s)
    e2e_schedule, e2e_s = e2e_choice(e2e_pipe_s, e2e_serial_s, pipelinable)
    e2e_value = aggregate_tokens_per_s(tokens, Ke, world, e2e_s)
    e2e_serial = aggregate_tokens_per_s(tokens, Ke, world, e2e_serial_s)
    e2e_pipe = aggregate_tokens_per_s(tokens, Ke, world, e2e_pipe_s)

    per_call, cands, launches = {}, [], 0
    for c, ms, ktimes in zip(calls, per_call_ms, kt):
        names = ["decode_kernel"] if c.form == "decode" else kernel_names(c.form, c.dtype, c.d, len(ktimes))
        launches += len(names) * c.steps
        s_call = ms / 1e3
        a = c.algorithmic_bytes()
        entry = {"us": round(ms * 1e3, 2), "GB_s": round(a / s_call / 1e9, 1),
                 "frac_hbm": round(a / s_call / 1e9 / peak, 4), "share": round(ms / step_ms, 3), "kernels": []}
        for i, (kn, kms) in enumerate(zip(names, ktimes)):
            kb = c.kernel_bytes(kn)
            entry["kernels"].append({"kernel": kn, "us": round(kms * 1e3, 2),
                                     "GB_s": round(kb / (kms / 1e3) / 1e9, 1) if kb else None,
                                     "frac_hbm": round(kb / (kms / 1e3) / 1e9 / peak, 4) if kb else None})
            if kb:
                cands.append((kms * c.steps, kms, c, kn, i, kb))
        per_call[f"{c.name}/{c.form}"] = entry

    # roofline of the dominant kernel: the one with the largest time in the
    # step, its algorithmic bytes over its own timed duration
    if not cands:
        raise SystemExit(f"no kernel of case {case} has algorithmic bytes: unknown kernel labels {per_call}")
    _, dom_ms, dom_call, dom_kernel, di, dom_bytes = max(cands, key=lambda x: x[0])
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    dtypes = sorted({c.dtype for c in calls})
    out = {
        "value": value,
        "unit": "tokens/s",
        "ms_per_step": step_ms,
        "dtype": dtypes[0] if len(dtypes) == 1 else "+".join(dtypes),
        "config": {"workload": CASE_TEXT[case] + (f" (scaled to {heads} heads)" if heads else ""),
                   "calls": [f"{c.name}: B={c.B} H={c.H} N={c.N} d={c.d} {c.dtype} {c.form}" for c in calls],
                   "global_batch": sum(c.B for c in calls) * world,
                   "seq_len": max(c.N for c in calls), "parallelism": f"dp{world}",
                   "l2": "flushed before every call (256 MiB write)",
                   "launch": "one CUDA graph per call" + (" (decode: 1024 steps in one graph)"
                                                          if any(c.form == "decode" for c in calls) else ""),
                   "tokens_per_step_per_gpu": tokens},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "serial_value": e2e_serial, "pipelined_value": e2e_pipe if pipelinable else None,
                "schedule": e2e_schedule,
                "mode": ("value = the faster of two schedules of the same copies and calls: pipelined (copies in "
                         "on one stream, the calls on another, copies out on a third, device tensors "
                         "double-buffered, so step i+1's inputs load while step i computes and copies out) and "
                         "serial (every copy and call of a step back to back on one stream)"
                         if pipelinable else
                         "per decode step: its token copied in, the step, its output copied out")},
        "gpu_launches": launches * K,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": recorded_traffic(dom_call.name, dom_call.dtype, f"{dom_call.form}/{di}"),
                     "kernel": f"{dom_kernel} (kernel {di} of {dom_call.name}/{dom_call.form})",
                     "kernel_us": round(dom_ms * 1e3, 2), "algorithmic_bytes": dom_bytes},
        "per_call": per_call,
    }
    if bad_flags:
        out["error_flags"] = bad_flags
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(calls, min_seconds=10.0 if case == HEADLINE else 3.0)
    return out


def run_ours(args, rank, world, local_rank):
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    from kernelized_linear_attention_phi_b200 import build as build_mod
    if rank == 0 or world == 1:
        build_mod.build()
    if world > 1:
        torch.distributed.barrier()
    peaks = load_peaks()
    peak = peaks.get("hbm_gbs", 6650.0)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    sampler = ClockSampler(device)
    sampler.start()
    try:
        head = measure_case(args.case, args, rank, world, device, flush, sampler, peak, args.scale_heads)
        torch.cuda.empty_cache()  # the case's buffers are released once it returns
        others = {}
        if not args.no_configs:
            for case in CASES:
                if case != args.case:
                    others[case] = measure_case(case, args, rank, world, device, flush, sampler, peak)
                    torch.cuda.empty_cache()
    finally:
        sampler.stop()
    result = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
              "warmup": max(args.warmup, 3), "ms_per_step": head["ms_per_step"], "higher_is_better": True,
              "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"], "data": "synthetic"}
    for key in ("config", "e2e", "gpu_launches", "roofline", "per_call", "cpu_baseline", "error_flags"):
        if key in head:
            result[key] = head[key]
    result["roofline"]["peak_source"] = peaks.get("_src")
    result["clocks"] = sampler.summary()
    if others:
        result["per_config"] = others
    bad = {k: v for k, v in [(args.case, head.get("error_flags"))] + [(c, o.get("error_flags"))
                                                                        for c, o in others.items()] if v}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    if bad:
        raise SystemExit(f"library error flags set during the run: {bad}")


def library_source_hash():
    """Hash of the library's CUDA sources: recorded DRAM traffic counts only
    for the kernels it was measured on."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kernelized_linear_attention_phi_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, dtype, key):
    """DRAM bytes (read + written) of one launch of a call's kernel
    ("causal/2": kernel 2 of the causal call) from the ncu launch list in
    profiles/traffic.json; None when none was taken for this workload and
    key, or the kernels changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_hash") != library_source_hash():
        return None
    return rec.get("bytes", {}).get(f"{workload}/{dtype}/{key}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        d["_src"] = "measured (MEASURED_PEAKS.json)"
        return d
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "_src": "fallback"}


# ---------------------------------------------------------------------------
# The oracle on the host cores (CPU baseline and reference arm)
# ---------------------------------------------------------------------------

def _blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return 1


# Tokens of one head the oracle's sample takes per call: all of them where
# the oracle's form is a few matrix products, a prefix of the sequence where
# it is a per-token loop (causal, prefix mask), the first steps of decode.
SAMPLE_TOKENS = {"noncausal": None, "causal": 4096, "prefix": 2048, "decode": 256,
                 "noncausal_bwd": 1024, "causal_bwd": 1024}


def oracle_sample(call_specs):
    """Runs the oracle, as it stands, on one head of each call (sequence 0,
    head 0; a prefix of the tokens where SAMPLE_TOKENS says so). Returns
    (seconds, tokens), tokens counted like the GPU step (B*N per
    full-sequence call, sequences x steps for decode) in the proportion of
    the work sampled: one head of H, n of N tokens, t of T steps."""
    import oracle
    total_t, tokens = 0.0, 0.0
    for spec in call_specs:
        form, phi, normalize, H = spec["form"], spec["phi"], spec["normalize"], spec["H"]
        Q, K, V = spec["Q"], spec["K"], spec["V"]
        n = Q.shape[0]
        t0 = time.perf_counter()
        if form == "noncausal":
            oracle.noncausal(Q, K, V, phi, normalize)
        elif form == "causal":
            oracle.causal(Q, K, V, phi, normalize)
        elif form == "prefix":
            oracle.prefix_mask(Q, K, V, spec["m"], phi, normalize)
        elif form == "decode":
            S, z = spec["S"], spec["z"]
            for t in range(n):
                _, S, z = oracle.decode_step(S, z, Q[t], K[t], V[t], phi, normalize)
        else:
            oracle.backward_dense(Q, K, V, spec["G"], form[:-4], None, phi, normalize)
        total_t += time.perf_counter() - t0
        if form == "decode":
            tokens += spec["B"] * n / H
        else:
            tokens += spec["B"] * spec["N"] * (n / spec["N"]) / H
    return total_t, tokens


def sample_specs(calls_or_cases):
    """The oracle's inputs for each call: head 0 of sequence 0, exact fp64
    copies of the GPU inputs (or, for the reference arm, of the same seeded
    inputs drawn on the host)."""
    specs = []
    f = lambda t: t.detach().to(torch.float64).cpu().numpy()
    for c in calls_or_cases:
        n = SAMPLE_TOKENS[c.form] or c.N
        spec = {"form": c.form, "phi": c.phi, "normalize": c.normalize, "H": c.H, "B": c.B, "N": c.N}
        if c.form == "decode":
            n = min(n, c.steps)
            spec.update(Q=f(c.qs[:n, 0, 0, 0]), K=f(c.ks[:n, 0, 0, 0]), V=f(c.vs[:n, 0, 0, 0]),
                        S=f(c.S[0, 0]), z=f(c.z[0, 0]))
            spec["N"] = c.steps
        else:
            n = min(n, c.N)
            spec.update(Q=f(c.q[0, 0, :n]), K=f(c.k[0, 0, :n]), V=f(c.v[0, 0, :n]))
            if c.form == "prefix":
                spec["m"] = np.minimum(c.m[0, :n].cpu().numpy(), n - 1) if n < c.N else c.m[0].cpu().numpy()
            if c.form.endswith("_bwd"):
                spec["G"] = f(c.dout[0, 0, :n])
        specs.append(spec)
    return specs


def cpu_baseline(calls, min_seconds=10.0):
    """The oracle, as it is, on the host cores: repeated passes over a
    sample of the case until about `min_seconds` of CPU work."""
    specs = sample_specs(calls)
    total_t, total_tok, passes = 0.0, 0.0, 0
    while total_t < min_seconds:
        dt, tok = oracle_sample(specs)
        total_t += dt
        total_tok += tok
        passes += 1
    what = ", ".join(f"{c.name}/{c.form}: head 0 of {c.H}, "
                     + (f"{min(SAMPLE_TOKENS[c.form], c.steps)} of {c.steps} steps" if c.form == "decode"
                        else f"{min(SAMPLE_TOKENS[c.form] or c.N, c.N)} of {c.N} tokens")
                     for c in calls)
    return {"value": total_tok / total_t, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"oracle (numpy fp64) on {what}; {passes} passes, {total_t:.1f} s; tokens scaled by the "
                      f"share of the work sampled; Python loops single-threaded, BLAS calls may use the cores"}


class _HostCall:
    """The inputs of one call of a case drawn on the host (reference arm):
    one head of the workload from the same seeded generators, drawn by the
    host's generator (the same distributions and shapes; the values differ
    from the device's draw), only what the oracle's sample reads."""

    def __init__(self, wl, dtype, form, mask):
        self.wl, self.form, self.name = wl, form, wl.name
        self.B, self.H, self.N, self.d = wl.B, wl.H, wl.N, wl.d
        self.phi, self.normalize, self.dtype = wl.phi, wl.normalize, dtype
        n = SAMPLE_TOKENS[form] or wl.N
        if form == "decode":
            self.steps = wl.decode_steps
            n = min(n, self.steps)
            qs, ks, vs = W.decode_tokens(n, 1, 1, wl.d, wl.sigma, wl.seed + 1, dtype, "cpu")
            self.qs, self.ks, self.vs = qs, ks, vs
            _, k0, v0 = W.qkv(1, 1, wl.N, wl.d, wl.sigma, wl.seed, dtype, "cpu")
            import oracle
            S, z = oracle.kv_summary(k0[0, 0].double().numpy(), v0[0, 0].double().numpy(), wl.phi)
            self.S, self.z = torch.from_numpy(S)[None, None], torch.from_numpy(z)[None, None]
        else:
            q, k, v = W.qkv(1, 1, wl.N, wl.d, wl.sigma, wl.seed, dtype, "cpu")
            self.q, self.k, self.v = q, k, v
            if form == "prefix":
                self.m = (W.prefix_mask_uniform(wl.B, wl.N, wl.seed, "cpu") if mask == "uniform"
                          else W.prefix_mask_arange(wl.B, wl.N, "cpu"))
            if form.endswith("_bwd"):
                self.dout = W.upstream_grad(1, 1, wl.N, wl.d, wl.seed, dtype, "cpu")


def run_reference(args, rank, world):
    if rank != 0:
        return
    calls = [_HostCall(W.WORKLOADS[w], dt, form, mask) for w, dt, form, mask in CASES[args.case]]
    specs = sample_specs(calls)
    for _ in range(args.warmup):
        oracle_sample(specs)
    total, tokens = 0.0, 0.0
    for _ in range(args.steps):
        dt, tok = oracle_sample(specs)
        total += dt
        tokens += tok
    value = tokens / total
    cores = _blas_threads()
    what = ", ".join(f"{c.name}/{c.form}: head 0 of {c.H}, "
                     + (f"{min(SAMPLE_TOKENS[c.form], c.steps)} of {c.steps} steps" if c.form == "decode"
                        else f"{min(SAMPLE_TOKENS[c.form] or c.N, c.N)} of {c.N} tokens") for c in calls)
    sample = (f"oracle (numpy fp64) per step on {what}; tokens scaled by the share of the work sampled")
    print(json.dumps({
        "impl": "reference", "metric": METRIC,
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": CASE_TEXT[args.case] + " (inputs; the oracle computes in fp64)",
                   "global_batch": sum(c.B for c in calls), "seq_len": max(c.N for c in calls),
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def record_traffic(csv_path, case, scale):
    """Per kernel launch of the last complete step of `case` in an ncu launch
    list: dram__bytes_read.sum + dram__bytes_write.sum, times `scale` (a
    capture of a smaller problem scaled to the case's size by the units each
    kernel processes), stored per workload/dtype/call/kernel index."""
    import csv
    with open(csv_path) as f:
        rows = [r for r in csv.reader(f)]
    head = next(i for i, r in enumerate(rows) if r and r[0] == "ID")
    h = rows[head]
    ik, im, iv, iu = (h.index(c) for c in ("Kernel Name", "Metric Name", "Metric Value", "Metric Unit"))
    units = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    launches = {}
    for r in rows[head + 1:]:
        if len(r) <= iv or "la::" not in r[ik]:
            continue
        rec = launches.setdefault(int(r[0]), {"name": r[ik], "bytes": 0.0})
        if r[im] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            rec["bytes"] += float(r[iv].replace(",", "")) * units.get(r[iu], 1)
    seq = [launches[i] for i in sorted(launches)]
    out_bytes = {}
    for w, dt, form, mask in CASES[case]:
        # the last complete launch of this call in the list (the bench's
        # per-kernel timing replays each call in turn after the timed steps)
        wl = W.WORKLOADS[w]
        name = wl.name if form != "prefix" or mask == "uniform" else f"{wl.name}_{mask}"
        table = kernel_table(dt, wl.d)[form]
        found = None
        for start in range(len(seq) - 1, -1, -1):
            for count in sorted(table, reverse=True):
                names = kernel_names(form, dt, wl.d, count)
                if start + len(names) <= len(seq) and all(k in seq[start + n]["name"] for n, k in enumerate(names)):
                    found = (start, names)
                    break
            if found:
                break
        if not found:
            raise SystemExit(f"the launch list holds no complete {name}/{form} call")
        start, names = found
        for n in range(len(names)):
            out_bytes[f"{name}/{dt}/{form}/{n}"] = int(seq[start + n]["bytes"] * scale)
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            out = json.load(f)
    except Exception:
        out = {}
    if out.get("source_hash") != library_source_hash():
        out = {"source_hash": library_source_hash(), "bytes": {}}
    out["note"] = ("DRAM bytes read + written per kernel launch (workload/dtype/call/index in launch order) "
                   "from an ncu launch list (cold cache per kernel); valid for the CUDA sources with this "
                   "hash; launches of a reduced-size capture are scaled to the workload's size")
    out["bytes"].update(out_bytes)
    with open(path, "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)
    print(json.dumps(out_bytes))


def main():
    args = parse()
    if args.record_traffic:
        record_traffic(args.record_traffic, args.case, args.traffic_scale)
        return
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
