"""Host logic of bench.py: the cases one run measures (every workload of the
pages, the long-context step as the headline), the names it gives the
kernels of each call from the count the library's timing events report, and
the algorithmic bytes of each kernel. Checked on CPU."""

import json
import subprocess
import sys

import bench
from kernelized_linear_attention_phi_b200 import workloads as W


def test_one_run_covers_every_workload_with_the_long_step_as_headline():
    assert bench.HEADLINE == "long"
    assert bench.CASES["long"] == [("long_noncausal", "bf16", "noncausal", None),
                                   ("long_causal", "bf16", "causal", None)]
    covered = {w for calls in bench.CASES.values() for w, *_ in calls}
    assert {"single_head", "multi_head", "prefix_mask", "long_noncausal", "long_causal", "decode"} <= covered
    assert ("multi_head", "f32", "causal", None) in bench.CASES["multi_head_f32"]
    assert [c[3] for c in bench.CASES["prefix_mask"] + bench.CASES["prefix_mask_arange"]] == ["uniform", "arange"]
    assert set(bench.CASE_TEXT) == set(bench.CASES)
    assert W.WORKLOADS["decode"].decode_steps == 1024


def test_kernel_names_follow_the_count_of_launches():
    kn = bench.kernel_names
    assert kn("noncausal", "bf16", 64, 1) == ["tc_noncausal_cluster_kernel"]
    assert kn("noncausal", "bf16", 64, 3) == ["tc_kv_kernel", "kv_reduce_balanced_kernel", "tc_readout_kernel"]
    assert kn("causal", "bf16", 128, 3) == ["tc_kv_kernel", "state_scan_kernel", "tc_sweep"]
    assert kn("causal", "bf16", 64, 2) == ["tc_kv_kernel", "tc_sweep"]
    assert kn("prefix", "bf16", 64, 3)[-1] == "tc_sweep"
    # fp32 at d = 64: the split-precision tensor-core kernel's modes; other
    # fp32 sizes and small d run on the CUDA cores
    assert kn("causal", "f32", 64, 3) == ["tc_f32_kernel<0", "state_scan_kernel", "tc_f32_kernel<1"]
    assert kn("noncausal", "f32", 64, 3) == ["tc_f32_kernel<0", "state_reduce_kernel", "tc_f32_kernel<2"]
    assert kn("prefix", "f32", 64, 4) == ["tc_f32_kernel<0", "bin_kernel", "state_scan_kernel", "tc_f32_kernel<3"]
    assert kn("prefix", "f32", 128, 4)[-1] == "chunked_kernel"
    assert kn("causal", "f32", 128, 3) == ["kv_partial_kernel", "state_scan_kernel", "chunked_kernel"]
    assert kn("noncausal", "bf16", 16, 3)[0] == "kv_partial_kernel"
    assert kn("noncausal", "f32", 16, 1) == ["noncausal_small_kernel"]  # short heads, d <= 32
    # a count the table does not know keeps neutral labels
    assert kn("causal", "bf16", 64, 7) == [f"kernel{i}" for i in range(7)]


def test_kernel_roles_cover_every_listed_kernel():
    for table in (bench.TC_KERNELS, bench.SIMT_KERNELS, bench.F32_TC_KERNELS):
        for by_count in table.values():
            for names in by_count.values():
                for n in names:
                    assert n in bench.KERNEL_ROLE, n


def test_kernel_bytes():
    """Algorithmic bytes per kernel: the KV pass reads K and V, a sweep reads
    Q, K, V and writes out, the readout reads Q and S, z and writes out, the
    gradient sweeps move their tensors once; scratch-only kernels have none."""
    B, H, N, d, e = 2, 8, 4096, 64, 2
    t = B * H * N * d * e
    st = B * H * (d * d + d) * 4
    kb = lambda form, k: bench.kernel_bytes(form, k, B, H, N, d, e)
    assert kb("causal", "tc_kv_kernel") == 2 * t
    assert kb("causal", "tc_sweep") == 4 * t
    assert kb("causal", "state_scan_kernel") == 0
    assert kb("noncausal", "tc_readout_kernel") == 2 * t + st
    assert kb("noncausal", "tc_noncausal_cluster_kernel") == 4 * t
    assert kb("noncausal", "noncausal_small_kernel") == 4 * t
    assert kb("prefix", "bin_kernel") == B * N * 4
    assert kb("decode", "decode_kernel") == 2 * st + 4 * B * H * d * e
    assert kb("noncausal_bwd", "tc_noncausal_cluster_kernel") == 2 * t
    assert kb("noncausal_bwd", "tc_bwd_q_kernel") == 3 * t
    assert kb("noncausal_bwd", "tc_bwd_kv_kernel") == 4 * t
    assert kb("noncausal_bwd", "kv_reduce_balanced_kernel") == 0
    assert kb("causal_bwd", "tc_bwd_causal_q_kernel") == 5 * t
    assert kb("causal_bwd", "tc_bwd_causal_kv_kernel") == 5 * t


def test_e2e_takes_the_faster_schedule():
    assert bench.e2e_choice(0.030, 0.040, True) == ("pipelined", 0.030)
    assert bench.e2e_choice(0.050, 0.040, True) == ("serial", 0.040)
    # decode: one schedule only, whatever the numbers say
    assert bench.e2e_choice(0.010, 0.040, False) == ("serial", 0.040)


def test_reference_arm_runs_on_the_host_and_prints_one_line():
    """--impl reference times the oracle on a sample of the headline case,
    on the host alone, and prints the contract's JSON line."""
    r = subprocess.run([sys.executable, bench.__file__, "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["unit"] == "tokens/s"
    assert rec["metric"] == bench.METRIC and rec["e2e"]["h2d_bytes_per_step"] == 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
