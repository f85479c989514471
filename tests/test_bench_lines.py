"""The bench's result lines, built from synthetic measurements on the CPU: the keys every line
carries, the throughput and roofline arithmetic, and end-to-end figures that move host bytes."""
import json

import pytest

import bench
import synth

REQUIRED = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "clocks", "e2e", "gpu_launches"}
PEAKS = {"hbm_gbs": 6551.0, "bf16_tflops": 1708.8}
CLOCKS = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 4}


def _check_common(line, workload):
    assert REQUIRED <= set(line)
    assert line["config"]["workload"] == workload
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    e2e = line["e2e"]
    assert e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert e2e["value"] != line["value"]  # measured on its own, not a copy of the device figure
    json.dumps(line, allow_nan=False)  # one plain JSON line: no NaN, nothing unserialisable


def test_decode_line_throughput_and_roofline():
    w = synth.WORKLOADS["decode80b"]
    args = bench.parse([])
    K = args.steps
    step_bytes = 1_035_829_248
    r = dict(ms=23.0, e2e_ms=23.4, kern_us=[1140.0], step_bytes=step_bytes, graph=True, uniq=[10.0] * 48,
             clocks=CLOCKS, gpu_launches=K, flags=0)
    line = bench.decode_line(args, w, 1, r, 1, PEAKS, "measured", None)
    _check_common(line, "decode80b")
    assert line["value"] == pytest.approx(K / 0.023, rel=1e-4)  # one token per step
    assert line["ms_per_step"] == pytest.approx(23.0 / K, rel=1e-3)
    rf = line["roofline"]
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s" and rf["peak"] == 6551.0
    assert rf["achieved"] == pytest.approx(step_bytes / 1140e-6 / 1e9, rel=1e-4)
    assert rf["frac"] == pytest.approx(rf["achieved"] / 6551.0, rel=1e-3)
    # dram bytes of one 48-layer launch: the per-layer capture times the layers
    assert rf["traffic"] == 21_664_640 * 48
    assert line["e2e"]["h2d_bytes_per_step"] == 2048 * 2  # one bf16 token in, one out
    assert line["e2e"]["value"] == pytest.approx(K / 0.0234, rel=1e-4)


def test_decode_line_traffic_unknown_for_other_stacks():
    w = synth.WORKLOADS["decode35b"]
    args = bench.parse(["--workload", "decode35b"])
    r = dict(ms=30.0, e2e_ms=31.0, kern_us=[1500.0], step_bytes=10**9, graph=True, uniq=[8.0] * 40,
             clocks=CLOCKS, gpu_launches=args.steps, flags=0)
    line = bench.decode_line(args, w, 8, r, 1, PEAKS, "measured", None)
    assert line["roofline"]["traffic"] is None
    assert "40-layer" in line["roofline"]["kernel"]
    assert line["value"] == pytest.approx(8 * args.steps / 0.030, rel=1e-4)


def test_prefill_flops_by_hand():
    # 2·m·n·k per matrix product: router 4096 x 513 x 2048; gate and up of 10 pairs per token
    # and of the shared expert (4096 x 1024 x 2048 each); down 4096·10 x 2048 x 512 and 4096 x
    # 2048 x 512
    router, gateup, down = bench.prefill_flops(synth.WORKLOADS["prefill"], 4096)
    assert router == 8_606_711_808
    assert gateup == 171_798_691_840 + 17_179_869_184
    assert down == 85_899_345_920 + 8_589_934_592


def test_prefill_line_throughput_and_roofline():
    w = synth.WORKLOADS["prefill"]
    args = bench.parse(["--workload", "prefill", "--steps", "10", "--warmup", "3"])
    r = dict(ms=7.3, e2e_ms=7.8, kern_us=[95.0, 53.5, 330.5, 251.7, 13.8], tokens_per_expert=(80.0, 48, 112),
             clocks=CLOCKS, flags=0)
    line = bench.prefill_line(args, w, 4096, r, 1, PEAKS, "measured", None)
    _check_common(line, "prefill")
    assert line["value"] == pytest.approx(4096 * 10 / 0.0073, rel=1e-4)
    rf = line["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s"
    assert rf["flops_per_launch"] == 188_978_561_024
    assert rf["achieved"] == pytest.approx(188_978_561_024 / 330.5e-6 / 1e12, rel=1e-3)
    assert rf["frac"] == pytest.approx(rf["achieved"] / 1708.8, rel=1e-3)
    assert line["e2e"]["h2d_bytes_per_step"] == 4096 * 2048 * 2


def test_pool_line_end_to_end_moves_bytes():
    w = synth.WORKLOADS["pool_int4"]
    args = bench.parse(["--workload", "pool_int4"])
    K = args.steps
    stats = {"hits": 700, "lookups": 1000, "h2d_bytes": 123}
    r = dict(K=K, ms=3.9, e2e_ms=4.1, hit_rate_all=0.685, hit_rate_timed=0.695, stats=stats, h2d_timed=10**8,
             zipf_s=1.0, clocks=CLOCKS, io_bytes=2048 * 2, flags=0)
    line = bench.pool_line(args, w, r, 1)
    _check_common(line, "pool_int4")
    assert line["value"] == pytest.approx(K / 0.0039, rel=1e-4)
    assert line["e2e"]["value"] == pytest.approx(K / 0.0041, rel=1e-4)
    assert line["config"]["n_slots"] == w.n_slots
