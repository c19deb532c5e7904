"""Host-side pieces of the benchmark that need no GPU: the algorithmic byte and FLOP models the
roofline fractions divide by, checked against sums written out by hand from their definitions, the
clock-record parsing, and the rule that a stored DRAM-traffic figure is only reported for the
workload it was taken on."""
import bench
from dynamic_block_sparse_proxy_b200 import workloads as W


def test_select_bytes_is_k_qlast_pe_q_and_index():
    """Llama geometry at 128k with 16 Pooled-Estimation heads and 8,298,280 selected pairs: K of 8
    kv-heads, the last 128 queries of 32 heads, all of Q of the 16 PE heads (bf16, d = 128) and the
    int32 index (row_ptr of N_b + 1 entries per head, one column per pair)."""
    w = W.WORKLOADS["llama8b_128k"]
    k = 8 * 131072 * 128 * 2
    q_last = 32 * 128 * 128 * 2
    q_pe = 16 * 131072 * 128 * 2
    index = 4 * (32 * 1025 + 8298280)
    assert k + q_last + q_pe + index == 839679264
    assert bench.select_bytes(w, 16, 8298280) == 839679264.0
    # a ragged length counts the partial last block in row_ptr
    r = W.WORKLOADS["tiny_1h_4k"]
    rr = type(r)(**{**r.__dict__, "n": 4000})
    assert bench.select_bytes(rr, 0, 10) == 4000 * 128 * 2 + 128 * 128 * 2 + 4 * (33 + 10)  # N_b = 32


def test_attn_flops_is_two_full_tile_products_per_pair():
    # QK^T and PV of a 128 x 128 tile with d = 128, two FLOPs per multiply-add
    assert bench.attn_flops(1) == 2 * 2 * 128 * 128 * 128
    assert bench.attn_flops(8298280) == 8298280 * 8388608


def test_clock_summary_median_max_and_reasons():
    lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n",
        "0, 1905, 1965, 995.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "0, 1890, 1965, 998.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "garbage line\n",
        "0, [N/A], 1965, 10.0, 0x0, Not Active, Not Active, Not Active, Not Active\n",
    ]
    s = bench.ClockSampler.summarise(lines)
    assert s["sm_mhz"] == 1905.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    hot = bench.ClockSampler.summarise(["1, 1500, 1965, 900, 0x48, Active, Active, Not Active, Not Active\n"])
    assert hot["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    assert bench.ClockSampler.summarise([])["sm_mhz"] is None


def test_stored_traffic_only_for_its_own_workload():
    assert bench.attn_traffic(W.WORKLOADS["llama8b_32k"]) is None
    assert bench.select_traffic(W.WORKLOADS["qwen7b_128k"]) is None
