"""Host-side arithmetic of bench.py, checked without a GPU: the kernel count it claims per layer
call against the launch lists taken with ncu on a B200 (profiles/launches_*.md), and the layer's
algorithmic work against the roofline table's figures for the Mixtral- and DeepSeek-V3-shaped
layers."""
import bench
from synth import workloads as W


def test_kernel_count_per_layer_call_matches_the_launch_lists():
    # V3 prefill: route_tc, two binary64 passes, refinement, histogram, scan, scatter, row copy,
    # routed GEMM1 and GEMM2, shared GEMM1 and GEMM2, combine
    assert bench.launches_per_step(W.get("deepseek_v3_prefill")) == 13
    # skewed capacity: logits GEMM, two passes, refinement, capacity, gates, histogram, scan,
    # scatter, row copy, GEMM1, GEMM2, combine
    assert bench.launches_per_step(W.get("skewed_capacity")) == 13
    # Mixtral-shaped: the V3 sequence without the shared experts
    assert bench.launches_per_step(W.get("mixtral_8x7b")) == 11


def test_expert_parallel_kernel_count_adds_the_exchange_and_barriers():
    w = W.get("deepseek_v3_prefill")
    per_rank = bench.ep_launches_per_rank(w, 2048, 8, False)
    # the single-device sequence without its scatter and row copy, plus the local histogram, scan
    # and scatter, the count publish and the row push
    assert per_rank == bench.launches_per_step(w) - 2 + 3 + 2
    assert bench.ep_launches_per_rank(w, 2048, 8, True) == per_rank + 4


def test_layer_work_matches_the_roofline_table():
    w = W.get("mixtral_8x7b")
    flops, nbytes = bench.layer_work(w, w.n * w.top_k, w.n_routed)
    assert abs(flops / 2.886e12 - 1) < 1e-3 and abs(nbytes / 2.89e9 - 1) < 2e-3
    w = W.get("deepseek_v3_prefill")
    flops, nbytes = bench.layer_work(w, w.n * w.top_k, w.n_routed)
    assert abs(flops / 13.05e12 - 1) < 1e-3 and abs(nbytes / 23.1e9 - 1) < 2e-3
