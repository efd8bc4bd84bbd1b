"""Host logic of bench.py that mirrors the library's dispatch: the kernels
each call of a workload launches (the labels of the per-kernel roofline),
the block count of the chunked forms and when the KV pass scans the block
states inside its clusters. Checked on CPU against the figures the dispatch
is written from."""

import bench
from kernelized_linear_attention_phi_b200 import workloads as W


def test_block_count_follows_the_block_plan():
    # one wave of 2 x 148 CTAs, blocks of at least 256 tokens in multiples of 128
    assert bench.block_count(W.WORKLOADS["multi_head"]) == 16      # 16 heads x 4096: 256-token blocks
    assert bench.block_count(W.WORKLOADS["prefix_mask"]) == 4      # 64 heads x 2048: 512-token blocks
    assert bench.block_count(W.WORKLOADS["long_causal"]) == 9      # d = 128, one CTA per SM


def test_in_cluster_scan_takes_two_blocks_per_cta_when_one_would_not_fit():
    wl = W.WORKLOADS["multi_head"]
    # 16 heads x 16 blocks: 16 clusters of 16 exceed the 14 a B200 holds, 16
    # clusters of 8 (two blocks per CTA) fit the 33
    assert bench.scan_in_cluster(wl)
    k = bench.call_kernels(wl, "bf16")
    assert k["causal"] == ["tc_kv_kernel", "tc_sweep"]
    assert k["prefix"] == ["tc_kv_kernel", "bin_kernel", "tc_sweep"]
    assert k["causal_bwd"] == ["tc_kv_kernel", "tc_bwd_causal_q_kernel", "state_scan_kernel",
                               "tc_bwd_causal_kv_kernel"]
    assert k["noncausal"] == ["tc_noncausal_cluster_kernel"]
    assert k["noncausal_bwd"] == ["tc_noncausal_cluster_kernel", "tc_bwd_q_kernel", "kv_reduce_balanced_kernel",
                                  "tc_bwd_kv_kernel"]


def test_long_and_fp32_workloads_keep_the_separate_kernels():
    k = bench.call_kernels(W.WORKLOADS["long_causal"], "bf16")  # d = 128: no in-cluster scan
    assert k["causal"] == ["tc_kv_kernel", "state_scan_kernel", "tc_sweep"]
    k = bench.call_kernels(W.WORKLOADS["long_noncausal"], "bf16")  # 64 heads: the balanced split
    assert k["noncausal"] == ["tc_kv_kernel", "kv_reduce_balanced_kernel", "tc_readout_kernel"]
    assert bench.call_kernels(W.WORKLOADS["multi_head"], "f32") == bench.CALL_KERNELS_F32


def test_kernel_roles_cover_every_listed_kernel():
    for table in (bench.CALL_KERNELS, bench.CALL_KERNELS_F32):
        for names in table.values():
            for n in names:
                assert any(n.startswith(r) for r in bench.KERNEL_ROLE), n


def test_kernel_bytes_of_the_gradient_calls():
    """Algorithmic bytes per kernel of the gradient calls: the KV summary
    reads K and V (whether the balanced KV pass or the cluster kernel without
    its readout forms it), the query side Q, dO and dq (causal: also K, V),
    the key side K, V, dk, dv (causal: also Q); reductions move scratch only."""
    wl = W.WORKLOADS["multi_head_bwd"]
    t = wl.B * wl.H * wl.N * wl.d * 2

    class S:  # the fields kernel_bytes reads
        B, H, N, d, elem = wl.B, wl.H, wl.N, wl.d, 2
    kb = lambda call, k: bench.Step.kernel_bytes(S, call, k)
    assert kb("noncausal_bwd", "tc_noncausal_cluster_kernel") == 2 * t
    assert kb("noncausal_bwd", "tc_kv_kernel") == 2 * t
    assert kb("noncausal_bwd", "tc_bwd_q_kernel") == 3 * t
    assert kb("noncausal_bwd", "tc_bwd_kv_kernel") == 4 * t
    assert kb("noncausal_bwd", "kv_reduce_balanced_kernel") == 0
    assert kb("causal_bwd", "tc_bwd_causal_q_kernel") == 5 * t
    assert kb("causal_bwd", "tc_bwd_causal_kv_kernel") == 5 * t
    assert kb("noncausal", "tc_noncausal_cluster_kernel") == 4 * t

