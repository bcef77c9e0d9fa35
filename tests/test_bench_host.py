"""Host-side arithmetic of the benchmark (CPU): the algorithmic FLOP and byte
counts behind the roofline numbers, the clock-sample summary that decides
whether a run is valid, the recorded DRAM-traffic lookup and the option
tables that must mirror the library's constants."""
import json
import os

import numpy as np

import bench
import routed_expert_ffn_prefix_b200 as moe
import synth


def test_layer_accounting_by_hand_decode_all_experts_touched():
    cfg = synth.CONFIGS["qwen_decode_t512"]           # T=512, H=4096, E=512, I=1024, k=10
    acc = bench.layer_accounting(cfg, np.full(cfg.E, 10))
    assert acc["touched"] == 512
    assert acc["flops"] == 6.0 * 10 * 4096 * 1024 * 512
    w = 512 * 3 * 4096 * 1024 * 2                     # gate/up (2I) + down (I) columns, bf16
    assert acc["layer_bytes"] == w + 512 * 4096 * 2 + 4096 * 512 * 4 + 512 * 4096 * 2
    # the gate/up kernel: weights once, x once, h written once
    assert acc["gate_up_bytes"] == 512 * 4096 * 2048 * 2 + 512 * 4096 * 2 + 512 * 10 * 1024 * 2
    assert acc["gate_up_bytes"] == 8_604_614_656


def test_layer_accounting_counts_only_touched_experts_and_the_shared_one():
    cfg = synth.CONFIGS["ling_skewed_t4096"]          # T=4096, H=8192, E=256, I=2048, k=8, I_s=2048
    counts = np.zeros(cfg.E, np.int64)
    counts[:100] = 1
    acc = bench.layer_accounting(cfg, counts)
    assert acc["touched"] == 100
    H, I, Is, T = 8192, 2048, 2048, 4096
    assert acc["flops"] == 6.0 * 8 * H * I * T + 6.0 * H * Is * T
    assert acc["layer_bytes"] == 100 * 3 * H * I * 2 + 3 * H * Is * 2 + T * H * 2 + H * 256 * 4 + T * H * 2


def test_kernel_roofline_picks_the_binding_unit():
    """The gate/up kernel's roofline object: HBM-bound when its bytes take
    longer at the copy peak than its FLOPs at the sustained bf16 peak (the
    bf16 prefill shape), tensor-bound otherwise (the same shape on FP8
    weights: half the weight bytes, the same MMAs)."""
    pk = {"hbm_gbs": 6539.5, "bf16_tflops": 1606.0, "bf16_tflops_sustained": 1367.0}
    cfg = synth.CONFIGS["qwen_prefill_t8192"]         # T=8192, H=4096, E=512, I=1024, k=10
    counts = np.full(cfg.E, 160)
    flops = 4.0 * 8192 * 10 * 4096 * 1024
    bf = bench.layer_accounting(cfg, counts)
    assert bf["gate_up_flops"] == flops
    r = bench.kernel_roofline(bf, 1.5, pk, "measured", None)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6539.5
    assert abs(r["achieved"] - bf["gate_up_bytes"] / 1.5e-3 / 1e9) < 0.1
    mx = bench.layer_accounting(cfg, counts, mx=True)
    assert mx["gate_up_bytes"] == 512 * 4096 * 2048 * (1 + 1 / 32) + 8192 * 4096 * 2 + 81920 * 1024 * 2
    r = bench.kernel_roofline(mx, 2.0, pk, "measured", None)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == 1367.0
    assert abs(r["achieved"] - flops / 2.0e-3 / 1e12) < 0.1
    assert abs(r["frac"] - r["achieved"] / 1367.0) < 1e-3
    # decode: far below the ridge on either weight format
    dc = synth.CONFIGS["qwen_decode_t512"]
    assert bench.kernel_roofline(bench.layer_accounting(dc, np.full(dc.E, 10), mx=True), 1.1, pk, "m",
                                 None)["bound"] == "hbm"


def test_clock_summary_median_and_reasons():
    clk = bench.ClockSampler(0)

    class _Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    class _Thread:
        def join(self, timeout=None):
            pass

    clk.proc, clk.thread = _Done(), _Thread()
    clk.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1900, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1930, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    s = clk.stop()
    assert s["sm_mhz"] == 1930 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    clk.lines[0] = "0, 1500, 1965, 500.0, 0x8, Not Active, Active, Not Active, Not Active"
    assert "hw_thermal_slowdown" in clk.stop()["reasons"]


def test_recorded_traffic_follows_the_source_hash():
    path = os.path.join(bench.ROOT, "profiles", "gate_up_traffic.json")
    rec = json.load(open(path))
    got = bench.recorded_traffic("qwen_decode_t512")
    if rec["kernel_source_hash"] == bench.kernel_source_hash():
        assert got == rec["per_launch_bytes"]["qwen_decode_t512"]
    else:  # the GEMM sources changed since the capture: no traffic is reported
        assert got is None
    assert bench.recorded_traffic("tiny") is None
    # the scaled figure is the 64-expert capture times 512 / 64
    assert abs(rec["per_launch_bytes"]["qwen_decode_t512"] - 8 * rec["measured_64_experts_bytes"]["prof_decode_e64"]) < 8


def test_option_tables_mirror_the_library_constants():
    assert bench.TILES == {"auto": moe.TILES_AUTO, "small": moe.TILES_SMALL, "large": moe.TILES_LARGE,
                           "pair": moe.TILES_PAIR, "persistent": moe.TILES_PERSISTENT}
    assert bench.COMBINE == {"auto": moe.COMBINE_AUTO, "fused": moe.COMBINE_FUSED,
                             "separate": moe.COMBINE_SEPARATE}
    assert bench.SCORING == {"softmax": moe.SCORE_SOFTMAX, "softmax_select_bias": moe.SCORE_SOFTMAX_SELECT_BIAS,
                             "sigmoid": moe.SCORE_SIGMOID}


def test_throughput_is_weak_scaling_over_the_slowest_rank():
    # 4 ranks x 512 tokens x 10 steps in 20 ms (slowest rank) -> 1.024 M tokens/s
    assert bench.throughput(512, 4, 10, 20.0) == 512 * 4 * 10 / 0.020
