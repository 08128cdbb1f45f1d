"""The benchmark's roofline accounting (host logic, no GPU): the algorithmic
work it divides by a duration is the closed form of the method's work."""
import bench

PEAKS = {"hbm_gbs": 6551.0, "bf16_tflops": 1688.4, "bf16_tflops_sustained": 1400.0}
D, E, K, N = 2560, 64, 4, 1024


def test_prefill_flops_are_the_pages_mac_count():
    # "So what does it cost?": 10.49M multiply-accumulates per token in the
    # value path (2560 x 1024 per expert, top-4), i.e. 2 flop each.
    T = 4096
    stage = {"route": 28.0, "group": 27.0, "experts": 107.0, "combine": 12.0}
    r = bench.roofline("prefill", "tensor", T, D, E, K, N, 2, [64] * 4, stage, 2.7, 0.1576, PEAKS, "measured")
    assert r["algorithmic_flops_per_launch"] == 2 * 10_485_760 * T
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    # the dominant stage is the GEMM; its duration is the stage time minus the event pair
    assert r["kernel_us"] == round(107.0 - 2.7, 3)
    assert abs(r["achieved"] - 2 * 10_485_760 * T / ((107.0 - 2.7) * 1e-6) / 1e12) < 0.1
    assert abs(r["frac"] - r["achieved"] / PEAKS["bf16_tflops"]) < 1e-4
    assert abs(r["step"]["frac"] - 2 * 10_485_760 * T / (0.1576e-3) / 1e12 / PEAKS["bf16_tflops"]) < 1e-4


def test_decode_bytes_are_the_active_experts_weights():
    # Each distinct active expert's n x d bf16 weight once, plus x and v; the
    # step adds the fp32 router weight and bias.
    T, distinct = 8, [24, 22, 22, 26]
    stage = {"route": 8.0, "group": 2.6, "experts": 28.6, "combine": 2.6}
    r = bench.roofline("decode", "stream", T, D, E, K, N, 2, distinct, stage, 2.7, 0.0267, PEAKS, "measured")
    Dm = sum(distinct) / len(distinct)
    kernel = Dm * N * D * 2 + T * D * 2 + T * N * 2
    assert r["algorithmic_bytes_per_launch"] == int(kernel)
    assert r["step"]["algorithmic_bytes_per_step"] == int(kernel + E * D * 4 + E * 4)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - kernel / ((28.6 - 2.7) * 1e-6) / 1e9) < 0.1
    assert abs(r["step"]["frac"] - (kernel + E * D * 4 + E * 4) / 0.0267e-3 / 1e9 / PEAKS["hbm_gbs"]) < 1e-4


def test_traffic_only_for_the_source_it_was_measured_on(monkeypatch):
    T = 4096
    stage = {"experts": 107.0}
    monkeypatch.setattr(bench, "source_sha", lambda files: "0000000000000000")
    r = bench.roofline("prefill", "tensor", T, D, E, K, N, 2, [64], stage, 2.7, 0.15, PEAKS, "measured")
    assert r["traffic"] is None
