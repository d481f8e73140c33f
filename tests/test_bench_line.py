"""bench.py's JSON line, assembled from synthetic timings on the CPU: the contract's
keys are there and the roofline, e2e and per-kernel figures follow from the timings by
the stated arithmetic."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def fake_result(step_ms=1.5, e2e_ms=36.0):
    kernels = {"gemm_3072x3072": [0.055], "gemm_3072x9216": [0.133], "gemm_3072x14336": [0.200, 0.202],
               "gemm_14336x3072": [0.190], "gemm_ffn_up_gelu_requant": [0.213], "gemm_ffn_down_bf16": [0.186],
               "quantize_32768x3072": [0.1], "dequantize_32768x3072": [0.055], "kv_append_8192": [0.06],
               "kv_window_4x8192": [0.093], "amax_history_push": [0.007]}
    scores = {"kv_window_scores": 0.32, "window_then_bmm": 0.41, "kv_window_context": 0.32,
              "window_then_bmm_v": 0.38}
    return {"ms_per_step": step_ms, "e2e_ms": e2e_ms, "kernels": kernels, "launches": 520,
            "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []},
            "h2d": 637534208, "d2h": 1872769084, "scores": scores}


def test_line_has_the_contract_keys_and_consistent_figures():
    args = type("A", (), {"steps": 20, "warmup": 5})()
    line = bench.summarize(fake_result(), args, 1)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True and line["scaling"] == "weak"
    assert "workload" in line["config"] and "model" not in line["config"]
    flops = bench.gemm_flops()
    assert abs(line["value"] - flops / 1.5e-3 / 1e12) < 0.01
    assert abs(line["e2e"]["value"] - flops / 36e-3 / 1e12) < 0.01
    assert line["e2e"]["h2d_bytes_per_step"] > 0 and line["e2e"]["d2h_bytes_per_step"] > 0
    r = line["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    # the dominant launch, 8192 x 14336 x 3072, at its mean time against 4 x the burst bf16 peak
    dom = 2.0 * 8192 * 14336 * 3072 / (0.201e-3) / 1e12
    assert abs(r["achieved"] - dom) < 0.2
    assert abs(r["peak"] - 4.0 * bench.read_peaks()["bf16_tflops"]) < 0.1
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    assert r["frac"] < 1.0
    assert r["traffic"] is None or r["traffic"] > 0
    k = line["kernels"]["kv_window_4x8192"]
    assert abs(k["gbs"] - bench.alg_bytes()["kv_window_4x8192"] / 0.093e-3 / 1e9) < 0.1
    assert line["kernels"]["gemm_ffn_up_gelu_requant"]["tflops"] > 0
    n = line["next_rows"]["attention_side_dequant"]
    assert abs(n["speedup"] - 0.41 / 0.32) < 1e-3 and abs(n["context_speedup"] - 0.38 / 0.32) < 1e-3


def test_value_is_the_whole_job_over_replicas():
    args = type("A", (), {"steps": 20, "warmup": 5})()
    one = bench.summarize(fake_result(), args, 1)
    four = bench.summarize(fake_result(), args, 4)
    assert abs(four["value"] - 4 * one["value"]) < 0.05 and four["n_gpus"] == 4
