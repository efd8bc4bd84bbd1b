"""Throughput of the kernelized linear attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload multi_head] [--dtype bf16]

One step is one pass of every form of the path over one batch of the
workload: non-causal (KV summary + readout), causal (chunked), prefix mask
(queries binned by m_i) and one decode step on the state the non-causal pass
produced. The default workload is multi-head attention with B=2, H=8,
N=4096, d=64 (the lineartile quick-start shape), phi = relu+1, normalized,
bf16, chunk 64, m_i uniform in [0, N-1]. Other workloads (--workload) run
only the forms they are defined for.

Tokens counted per step: B*N for each full-sequence form plus B for a decode
step. ``value`` is tokens/s over all ranks (weak scaling: each rank runs its
own batch; the path has no exchange step, so there is no data-path
collective). Each library call is captured once into a CUDA graph and the
graphs are replayed. Timing: CUDA events between the calls of every step on
the launching stream, L2 flushed (a 256 MiB write) between steps outside the
events, W untimed warm-up steps, max over ranks. ``e2e`` repeats the step
through the plain API calls with pinned host inputs copied in and the
outputs copied back inside the timed region. ``roofline`` is the dominant
kernel's: after the timed steps every call is replayed again from a graph
captured with the library's per-kernel timing events (la_timing_enable), L2
flushed before each replay, and the kernel with the largest mean time has its
algorithmic bytes divided by that time.
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

# Kernels each library call launches on the bf16 tensor-core path, in launch
# order; kept in step with la_api.cu's dispatch and checked against the ncu
# launch list (--record-traffic matches them there).
CALL_KERNELS = {
    "noncausal": ["tc_kv_kernel", "kv_reduce_balanced_kernel", "tc_readout_kernel"],
    "causal": ["tc_kv_kernel", "state_scan_kernel", "tc_sweep"],
    "prefix": ["tc_kv_kernel", "bin_kernel", "state_scan_kernel", "tc_sweep"],
    "decode": ["decode_kernel"],
    "noncausal_bwd": ["tc_kv_kernel", "kv_reduce_balanced_kernel", "tc_bwd_q_kernel", "kv_reduce_balanced_kernel",
                      "tc_bwd_kv_kernel"],
    "causal_bwd": ["tc_kv_kernel", "state_scan_kernel", "tc_bwd_causal_q_kernel", "state_scan_kernel",
                   "tc_bwd_causal_kv_kernel"],
}
# The same on the fp32 (CUDA-core) path.
CALL_KERNELS_F32 = {
    "noncausal": ["kv_partial_kernel", "state_reduce_kernel", "readout_kernel"],
    "causal": ["kv_partial_kernel", "state_scan_kernel", "chunked_kernel"],
    "prefix": ["kv_partial_kernel", "bin_kernel", "state_scan_kernel", "chunked_kernel"],
    "decode": ["decode_kernel"],
    "noncausal_bwd": ["kv_partial_kernel", "state_reduce_kernel", "bwd_q_kernel", "state_reduce_kernel",
                      "bwd_kv_kernel"],
    "causal_bwd": ["kv_partial_kernel", "state_scan_kernel", "bwd_q_kernel", "state_scan_kernel", "bwd_kv_kernel"],
}


def call_kernels(wl, dtype):
    """The kernels of each call for this workload: the tables above, with the
    non-causal form as one thread-block-cluster kernel where la_noncausal
    takes that path (bf16, d = 64, B*H <= 33, N <= 8192; the non-causal
    gradient then forms its KV summary with it too), and without
    the block-state scan kernel where the KV pass scans in its clusters
    (scan_in_cluster)."""
    if dtype != "bf16":
        return CALL_KERNELS_F32
    out = dict(CALL_KERNELS)
    if wl.d == 64 and wl.B * wl.H <= 33 and wl.N <= 8192:
        out["noncausal"] = ["tc_noncausal_cluster_kernel"]
        # the gradient's KV summary: the same kernel without its readout
        out["noncausal_bwd"] = ["tc_noncausal_cluster_kernel"] + out["noncausal_bwd"][2:]
    if wl.d == 64 and scan_in_cluster(wl):
        # the KV pass scans the block states inside its clusters (causal,
        # prefix mask, causal gradients): no forward scan kernel
        out["causal"] = [k for k in out["causal"] if k != "state_scan_kernel"]
        out["prefix"] = [k for k in out["prefix"] if k != "state_scan_kernel"]
        out["causal_bwd"] = [k for i, k in enumerate(out["causal_bwd"]) if not (i == 1 and k == "state_scan_kernel")]
    return out


def scan_in_cluster(wl):
    """Whether the KV pass scans the block states in a cluster per head, as
    tc_kv.cu decides it: at most 16 blocks, and every head's cluster (one or
    two blocks per CTA) resident at once; a B200 holds 71 clusters of 4, 33
    of 8 and 14 of 16 at two CTAs per SM."""
    nblk, bh = block_count(wl), wl.B * wl.H

    def capacity(cs):
        return 296 if cs <= 1 else 148 if cs <= 2 else 71 if cs <= 4 else 33 if cs <= 8 else 14
    return nblk <= 16 and any(bh <= capacity(-(-nblk // bpc)) for bpc in (1, 2))


def block_count(wl):
    """Blocks per head of the chunked forms, as la_api.cu's block plan picks
    them (one wave of 148 SMs x 2 CTAs, blocks of at least 256 tokens, a
    multiple of 128)."""
    per_sm = 1 if wl.d == 128 else 2
    target = max(1, per_sm * 148 // (wl.B * wl.H))
    bt = max(256, -(-(-(-wl.N // target)) // 128) * 128)
    return -(-wl.N // bt)


# What each kernel does, for its algorithmic bytes (Step.kernel_bytes).
KERNEL_ROLE = {"tc_kv_kernel": "kv", "kv_partial_kernel": "kv", "kv_reduce_balanced_kernel": "reduce",
               "state_reduce_kernel": "reduce", "tc_readout_kernel": "readout", "readout_kernel": "readout",
               "state_scan_kernel": "scan", "tc_sweep": "sweep", "chunked_kernel": "sweep",
               "bin_kernel": "bin", "decode_kernel": "decode", "bwd_q_kernel": "bwd_q",
               "bwd_kv_kernel": "bwd_kv", "tc_bwd_q_kernel": "bwd_q", "tc_bwd_kv_kernel": "bwd_kv",
               "tc_bwd_causal_q_kernel": "bwd_q", "tc_bwd_causal_kv_kernel": "bwd_kv",
               "tc_noncausal_cluster_kernel": "fused"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="multi_head")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f32"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--record-traffic", metavar="NCU_CSV",
                    help="read an ncu launch list with dram__bytes_read.sum and "
                         "dram__bytes_write.sum of this workload's bench run and store "
                         "each call's DRAM bytes in profiles/traffic.json")
    return ap.parse_args()


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
            self._sample()
            time.sleep(0.01)

    def __enter__(self):
        if self.nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self.nv or not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples),
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b]}


# ---------------------------------------------------------------------------
# The step
# ---------------------------------------------------------------------------

class Step:
    """Device buffers and the four library calls of one step."""

    ALL_FORMS = ("noncausal", "causal", "prefix", "decode")

    def __init__(self, wl, dtype, seed, device, forms):
        from kernelized_linear_attention_phi_b200 import binding as la
        self.la = la
        self.forms = forms
        B, H, N, d = wl.B, wl.H, wl.N, wl.d
        self.wl, self.B, self.H, self.N, self.d = wl, B, H, N, d
        self.phi, self.normalize, self.chunk = wl.phi, wl.normalize, wl.chunk
        self.q, self.k, self.v = W.qkv(B, H, N, d, wl.sigma, seed, dtype, device)
        self.m = W.prefix_mask_uniform(B, N, seed, device)
        q1, k1, v1 = W.decode_tokens(1, B, H, d, wl.sigma, seed, dtype, device)
        self.q1, self.k1, self.v1 = q1[0].contiguous(), k1[0].contiguous(), v1[0].contiguous()
        self.out_nc = torch.empty_like(self.q)
        self.out_c = torch.empty_like(self.q)
        self.out_m = torch.empty_like(self.q)
        self.out_d = torch.empty_like(self.q1)
        if any(f.endswith("_bwd") for f in forms):
            self.dout = W.upstream_grad(B, H, N, d, seed, dtype, device)
            self.grads = {f: tuple(torch.empty_like(self.q) for _ in range(3)) for f in forms}
        self.S = torch.empty(B, H, d, d, dtype=torch.float32, device=device)
        self.z = torch.empty(B, H, d, dtype=torch.float32, device=device)
        desc = la._desc_of(self.q, self.phi, self.normalize)
        self.ws = {op: la.workspace(desc, op, self.chunk, device)
                   for op in ("noncausal", "causal", "prefix") + tuple(f for f in forms if f.endswith("_bwd"))}
        self.tokens = sum(B if f == "decode" else B * N for f in forms)
        self.elem = self.q.element_size()
        if "decode" in forms and "noncausal" not in forms:
            # the cached state the decode steps continue from: a prefill of N tokens
            la.la_kv_summary(self.k, self.v, self.S, self.z, self.phi)

    def calls(self):
        la = self.la
        table = {
            "noncausal": lambda: la.la_noncausal(self.q, self.k, self.v, self.out_nc, self.S, self.z,
                                                 self.phi, self.normalize, self.ws["noncausal"]),
            "causal": lambda: la.la_causal_chunked(self.q, self.k, self.v, self.out_c, self.chunk,
                                                   self.phi, self.normalize, self.ws["causal"]),
            "prefix": lambda: la.la_prefix_mask(self.q, self.k, self.v, self.m, self.out_m, self.chunk,
                                                self.phi, self.normalize, self.ws["prefix"]),
            "decode": lambda: la.la_decode_step(self.q1, self.k1, self.v1, self.S, self.z, self.out_d,
                                                self.phi, self.normalize),
            "noncausal_bwd": lambda: la.la_noncausal_backward(self.q, self.k, self.v, self.dout,
                                                              *self.grads["noncausal_bwd"], self.phi,
                                                              self.normalize, self.ws["noncausal_bwd"]),
            "causal_bwd": lambda: la.la_causal_backward(self.q, self.k, self.v, self.dout,
                                                        *self.grads["causal_bwd"], self.phi, self.normalize,
                                                        self.ws["causal_bwd"]),
        }
        return [(f, table[f]) for f in self.forms]

    def algorithmic_bytes(self):
        """Bytes each call must move at least: its inputs once and outputs once."""
        t = self.B * self.H * self.N * self.d * self.elem     # one [B,H,N,d] tensor
        st = self.B * self.H * (self.d * self.d + self.d) * 4  # fp32 (S, z)
        one = self.B * self.H * self.d * self.elem
        return {"noncausal": 4 * t + st, "causal": 4 * t, "prefix": 4 * t + self.B * self.N * 4,
                "decode": 2 * st + 4 * one, "noncausal_bwd": 7 * t, "causal_bwd": 7 * t}

    def kernel_bytes(self, call, kernel):
        """Algorithmic bytes of one kernel of a call: the method's tensors it
        must read or write once (Q, K, V, out, S, z, m). Scratch the library
        keeps between its kernels (partial and block-state records, the
        binning tables) is not counted, so a kernel that only moves scratch
        (the prefix scan over block states) has none."""
        t = self.B * self.H * self.N * self.d * self.elem
        st = self.B * self.H * (self.d * self.d + self.d) * 4
        one = self.B * self.H * self.d * self.elem
        role = KERNEL_ROLE.get(kernel)
        if call.endswith("_bwd"):
            # gradients: q, k, v, dout read and dq, dk, dv written once over
            # the sweeps (non-causal: q, dout -> dq; k, v -> dk, dv; causal:
            # q, k, v, dout -> dq; q, k, v -> dk, dv); the reductions of
            # (G, h) move scratch only
            causal = call == "causal_bwd"
            return {"kv": 2 * t, "fused": 2 * t, "bwd_q": (5 if causal else 3) * t,
                    "bwd_kv": (5 if causal else 4) * t}.get(role, 0)
        return {"kv": 2 * t, "reduce": st, "readout": 2 * t + st, "scan": 0, "sweep": 4 * t, "fused": 4 * t,
                "bin": self.B * self.N * 4, "decode": 2 * st + 4 * one}.get(role, 0)

    def host_io(self):
        full = [f for f in self.forms if f != "decode"]
        bwd = [f for f in self.forms if f.endswith("_bwd")]
        ins = ([self.q, self.k, self.v] if full else []) + ([self.m] if "prefix" in self.forms else []) \
            + ([self.q1, self.k1, self.v1] if "decode" in self.forms else []) + ([self.dout] if bwd else [])
        outs = []
        for f in self.forms:
            if f.endswith("_bwd"):
                outs += list(self.grads[f])
            else:
                outs.append({"noncausal": self.out_nc, "causal": self.out_c, "prefix": self.out_m,
                             "decode": self.out_d}[f])
        return ins, outs


def kernel_times(step, calls, flush, reps):
    """Per call: the mean duration (ms) of each kernel it launches, from the
    library's timing events over `reps` replays of a graph of the call."""
    la = step.la
    la.la_timing_enable(True)
    out = {}
    try:
        for name, fn in calls:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            acc = None
            for _ in range(reps):
                flush_l2(flush)
                g.replay()
                ms = la.la_timing_read()
                acc = ms if acc is None else [a + b for a, b in zip(acc, ms)]
            out[name] = [a / reps for a in acc]
            del g
    finally:
        la.la_timing_enable(False)
    return out


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
    wl = W.WORKLOADS[args.workload]
    dtype = args.dtype if args.dtype in wl.dtypes else wl.dtypes[0]
    forms = Step.ALL_FORMS if args.workload == "multi_head" else wl.forms
    step = Step(wl, dtype, rank_seed(wl, rank), device, forms)
    calls = step.calls()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    for _ in range(max(args.warmup, 3)):
        for _, fn in calls:
            fn()
    torch.cuda.synchronize()
    graphs = []
    for _, fn in calls:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        graphs.append(g)
    for _ in range(max(args.warmup, 3)):
        for g in graphs:
            g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)

    K = args.steps
    sampler = ClockSampler(device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # Every call starts with a cold L2 (a 256 MiB write between calls, outside
    # the events), so each call reads its inputs from HBM; a step's time is
    # the sum of its calls' times.
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(len(calls))] for _ in range(K)]
    with sampler:
        for i in range(K):
            for j, g in enumerate(graphs):
                flush_l2(flush)
                ev[i][j][0].record(stream)
                g.replay()
                ev[i][j][1].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    per_call = {name: 0.0 for name, _ in calls}
    total_ms = 0.0
    for i in range(K):
        for j, (name, _) in enumerate(calls):
            ms = ev[i][j][0].elapsed_time(ev[i][j][1])
            per_call[name] += ms
            total_ms += ms
    t_s = total_ms / 1e3

    # end to end through the public API: pinned host inputs in, outputs back
    ins, outs = step.host_io()
    h_ins = [t.cpu().pin_memory() for t in ins]
    h_outs = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in h_ins)
    d2h = sum(t.numel() * t.element_size() for t in h_outs)
    Ke = max(1, min(K, 50))
    e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Ke)]
    torch.cuda.synchronize()
    for i in range(Ke):
        flush_l2(flush)
        e_ev[i][0].record(stream)
        for d_t, h_t in zip(ins, h_ins):
            d_t.copy_(h_t, non_blocking=True)
        for _, fn in calls:
            fn()
        for h_t, d_t in zip(h_outs, outs):
            h_t.copy_(d_t, non_blocking=True)
        e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_s = sum(a.elapsed_time(b) for a, b in e_ev) / 1e3

    # each kernel's own duration: the calls replayed again from graphs
    # captured with the library's per-kernel timing events (an event node
    # between two kernels; the call-level numbers above come from graphs
    # without them), L2 flushed before every replay, averaged over the replays
    kt = kernel_times(step, calls, flush, max(3, min(K, 20)))

    # every call reports expired bounded waits in its workspace error word
    flags = {op: step.la.la_last_error(ws)[1] for op, ws in step.ws.items()}
    bad_flags = {op: f for op, f in flags.items() if f}

    t_s, e2e_s = max_over_ranks([t_s, e2e_s], device)
    value = aggregate_tokens_per_s(step.tokens, K, world, t_s)
    e2e_value = aggregate_tokens_per_s(step.tokens, Ke, world, e2e_s)

    peaks = load_peaks()
    peak = peaks.get("hbm_gbs", 6650.0)
    names = call_kernels(wl, dtype)
    per_kernel = {}
    for name in per_call:
        s_call = per_call[name] / 1e3 / K
        a = step.algorithmic_bytes()[name]
        entry = {"us": round(s_call * 1e6, 2), "GB_s": round(a / s_call / 1e9, 1),
                 "frac_hbm": round(a / s_call / 1e9 / peak, 3),
                 "share": round(per_call[name] / sum(per_call.values()), 3), "kernels": []}
        for i, ms in enumerate(kt.get(name, [])):
            kn = names[name][i] if i < len(names[name]) else f"kernel{i}"
            kb = step.kernel_bytes(name, kn)
            entry["kernels"].append({"kernel": kn, "us": round(ms * 1e3, 2),
                                     "GB_s": round(kb / (ms / 1e3) / 1e9, 1) if kb else None,
                                     "frac_hbm": round(kb / (ms / 1e3) / 1e9 / peak, 3) if kb else None})
        per_kernel[name] = entry

    # roofline of the dominant kernel: the (call, kernel) with the largest
    # time in the step, its algorithmic bytes over its own timed duration
    cands = [(ms, name, i) for name, lst in kt.items() for i, ms in enumerate(lst)
             if step.kernel_bytes(name, names[name][i] if i < len(names[name]) else "") > 0]
    dom_ms, dom, di = max(cands)
    dom_kernel = names[dom][di]
    dom_bytes = step.kernel_bytes(dom, dom_kernel)
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    result = {
        "metric": "tokens/sec (fwd, 1xB200) and % of HBM / bf16 tensor-core roofline per kernel",
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": max(args.warmup, 3),
        "ms_per_step": total_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype,
        "data": "synthetic",
        "config": {"workload": f"{wl.name}: B={wl.B} H={wl.H} N={wl.N} d={wl.d} {dtype} phi={wl.phi} "
                               f"normalize={int(wl.normalize)} chunk={wl.chunk}; step = "
                               + " + ".join({"noncausal": "noncausal", "causal": "causal",
                                             "prefix": "prefix mask (m uniform)",
                                             "decode": "1 decode step",
                                             "noncausal_bwd": "noncausal gradients",
                                             "causal_bwd": "causal gradients"}[f] for f in forms),
                   "global_batch": wl.B * world, "seq_len": wl.N, "parallelism": f"dp{world}",
                   "l2": "flushed between steps (256 MiB write)", "launch": "one CUDA graph per call",
                   "tokens_per_step_per_gpu": step.tokens},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": sum(len(names[n]) for n, _ in calls) * K,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": recorded_traffic(wl.name, dtype, f"{dom}/{di}"),
                     "kernel": f"{dom_kernel} (kernel {di} of la_{dom})",
                     "kernel_us": round(dom_ms * 1e3, 2), "peak_source": peaks.get("_src"),
                     "algorithmic_bytes": dom_bytes},
        "per_call": per_kernel,
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(step, heads=2)
    if bad_flags:
        result["error_flags"] = bad_flags
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    if bad_flags:
        raise SystemExit(f"library error flags set during the run: {bad_flags}")


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
    """DRAM bytes (read + write) of one call ("causal") or one of its kernels
    ("causal/2", by launch index) from the ncu capture in
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


def oracle_sample(q, k, v, m, q1, k1, v1, phi, normalize, heads, forms, dout=None):
    """Runs the oracle's forms on the first `heads` heads of sequence 0.
    Returns (seconds, tokens processed), tokens counted like the GPU step
    (B*N per full-sequence form, B per decode step) scaled by heads/H."""
    import oracle
    f = lambda t: t.detach().to(torch.float64).cpu().numpy()
    H = q.shape[1]
    Q, K, V = f(q[0, :heads]), f(k[0, :heads]), f(v[0, :heads])
    M = m[0].cpu().numpy()
    q1_, k1_, v1_ = f(q1[0, :heads, 0]), f(k1[0, :heads, 0]), f(v1[0, :heads, 0])
    G = f(dout[0, :heads]) if dout is not None else None
    N = Q.shape[1]
    t0 = time.perf_counter()
    for h in range(heads):
        S = z = None
        if "noncausal" in forms:
            _, S, z = oracle.noncausal(Q[h], K[h], V[h], phi, normalize)
        if "causal" in forms:
            oracle.causal(Q[h], K[h], V[h], phi, normalize)
        if "prefix" in forms:
            oracle.prefix_mask(Q[h], K[h], V[h], M, phi, normalize)
        if "decode" in forms:
            if S is None:
                S, z = oracle.kv_summary(K[h], V[h], phi)
            oracle.decode_step(S, z, q1_[h], k1_[h], v1_[h], phi, normalize)
        for fm in ("noncausal_bwd", "causal_bwd"):
            if fm in forms:
                oracle.backward_dense(Q[h], K[h], V[h], G[h], fm[:-4], None, phi, normalize)
    dt = time.perf_counter() - t0
    per_seq = sum(1 if fm == "decode" else N for fm in forms)
    return dt, per_seq * heads / H


def cpu_baseline(step, heads=2, min_seconds=10.0):
    """The oracle, as it is, on the host cores: repeated passes over a
    sample of heads until about `min_seconds` of CPU work."""
    total_t, total_tok, passes = 0.0, 0.0, 0
    while total_t < min_seconds:
        dt, tok = oracle_sample(step.q, step.k, step.v, step.m, step.q1, step.k1, step.v1,
                                step.phi, step.normalize, heads, step.forms, getattr(step, "dout", None))
        total_t += dt
        total_tok += tok
        passes += 1
    return {"value": total_tok / total_t, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"oracle (numpy fp64) on {heads} of {step.H} heads of sequence 0, forms "
                      f"{'+'.join(step.forms)}, N={step.N}, {passes} passes, {total_t:.1f} s; tokens "
                      f"scaled by heads/H; Python loops single-threaded, BLAS calls may use the cores"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = W.WORKLOADS[args.workload]
    dtype = args.dtype if args.dtype in wl.dtypes else wl.dtypes[0]
    forms = Step.ALL_FORMS if args.workload == "multi_head" else wl.forms
    q, k, v = W.qkv(1, wl.H, wl.N, wl.d, wl.sigma, wl.seed, dtype, "cpu")
    m = W.prefix_mask_uniform(1, wl.N, wl.seed, "cpu")
    q1, k1, v1 = (t[0] for t in W.decode_tokens(1, 1, wl.H, wl.d, wl.sigma, wl.seed, dtype, "cpu"))
    dout = W.upstream_grad(1, wl.H, wl.N, wl.d, wl.seed, dtype, "cpu")
    heads = 1
    for _ in range(args.warmup):
        oracle_sample(q, k, v, m, q1, k1, v1, wl.phi, wl.normalize, heads, forms, dout)
    total, tokens = 0.0, 0.0
    for _ in range(args.steps):
        dt, tok = oracle_sample(q, k, v, m, q1, k1, v1, wl.phi, wl.normalize, heads, forms, dout)
        total += dt
        tokens += tok
    value = tokens / total
    cores = _blas_threads()
    sample = (f"oracle (numpy fp64) on {heads} of {wl.H} heads of one sequence per step, forms "
              f"{'+'.join(forms)}, N={wl.N}; tokens scaled by heads/H")
    print(json.dumps({
        "impl": "reference",
        "metric": "tokens/sec (fwd, 1xB200) and % of HBM / bf16 tensor-core roofline per kernel",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{wl.name}: B={wl.B} H={wl.H} N={wl.N} d={wl.d} {dtype} inputs",
                   "global_batch": wl.B, "seq_len": wl.N, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def record_traffic(csv_path, workload, dtype):
    """Per call of the last complete step in an ncu launch list: the sum of
    dram__bytes_read.sum + dram__bytes_write.sum over the call's kernels."""
    import csv
    with open(csv_path) as f:
        rows = [r for r in csv.reader(f)]
    head = next(i for i, r in enumerate(rows) if r and r[0] == "ID")
    h = rows[head]
    ik, im, iv, iu = (h.index(c) for c in ("Kernel Name", "Metric Name", "Metric Value", "Metric Unit"))
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    launches = {}
    for r in rows[head + 1:]:
        if len(r) <= iv or "la::" not in r[ik]:
            continue
        rec = launches.setdefault(int(r[0]), {"name": r[ik], "bytes": 0.0})
        if r[im] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            rec["bytes"] += float(r[iv].replace(",", "")) * scale.get(r[iu], 1)
    seq = [launches[i] for i in sorted(launches)]
    forms = Step.ALL_FORMS if workload == "multi_head" else W.WORKLOADS[workload].forms
    names = call_kernels(W.WORKLOADS[workload], dtype)
    want = [(f, k) for f in forms for k in names[f]]
    for start in range(len(seq) - len(want), -1, -1):
        if all(k in seq[start + n]["name"] for n, (_, k) in enumerate(want)):
            break
    else:
        raise SystemExit("the launch list holds no complete step of this workload")
    per_call, per_kernel = {}, {}
    for n, (f, _) in enumerate(want):
        per_call[f] = per_call.get(f, 0.0) + seq[start + n]["bytes"]
        i = sum(1 for g, _ in want[:n] if g == f)  # the kernel's index within its call
        per_kernel[f"{f}/{i}"] = seq[start + n]["bytes"]
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            out = json.load(f)
    except Exception:
        out = {}
    if out.get("source_hash") != library_source_hash():
        out = {"source_hash": library_source_hash(), "bytes": {}}
    out["note"] = ("DRAM bytes read + written per library call (workload/dtype/call, summed over "
                   "the call's kernels) and per kernel (workload/dtype/call/index in launch order), "
                   "from an ncu launch list (cold cache per kernel); valid for the CUDA sources "
                   "with this hash")
    for f, b in per_call.items():
        out["bytes"][f"{workload}/{dtype}/{f}"] = int(b)
    for key, b in per_kernel.items():
        out["bytes"][f"{workload}/{dtype}/{key}"] = int(b)
    with open(path, "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)
    print(json.dumps(per_call))


def main():
    args = parse()
    if args.record_traffic:
        record_traffic(args.record_traffic, args.workload, args.dtype)
        return
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
