"""The bench line stays compact: the summary of every section, filled with numbers of the widths a
run produces, serialises to well under the size the line may take (the full numbers go to the
--details file)."""
import json

import bench


def _sections():
    sweep = [{"M": m, "gemm_us": 67.1234, "gemm_frac_hbm": 0.2134, "gemm_frac_fp4_peak": 0.5512,
              "act_quant_us": 9.1234, "fused_layer_us": 88.1234,
              "w4a16_layer_us": 33.1234 if m <= 64 else None} for m in (1, 16, 128, 2048)]
    overhead = {"B_vs_plain_mxfp4_pipeline": 0.0205123, "A_vs_gemm_on_prequantized_A": 0.153123,
                "two_kernel_B": 0.0205123}
    prefill = {"points": [{"M": m, "K": k, "N": n, "gemm_frac_fp4_peak": 0.7612, "overhead_B_transform": 0.0312,
                           "overhead_B_fused": 0.1812, "act_quant_frac_hbm": 0.5912}
                          for m in (4096, 16384) for k in (8192, 16384) for n in (8192, 28672)]}
    qwen3 = {"points": [{"M": m, "layer_us": 983.123, "layer_fused_qkv_gateup_us": 976.123, "swiglu_fused_us": 468.12,
                         "swiglu_two_step_us": 1226.12} for m in (1, 8, 64, 4096)]}
    moe = {"points": [dict({"proj": p, "T": t, "grouped_gemm_us": 155.123, "grouped_gemm_frac_hbm": 0.4812,
                            "grouped_gemm_frac_fp4_peak": 0.4112},
                           **({"combine_us": 50.1, "combine_frac_hbm": 0.9212} if p == "down" else {}))
                      for p in ("gate_up", "down") for t in (64, 1024, 8192)]}
    prep = {"us": 35.6123, "frac_hbm": 0.6412}
    ceiling = [{"bytes": 21233664, "us": 5.3, "gbs": 3988.12}, {"bytes": 679477248, "us": 103.7, "gbs": 6550.12}]
    flip = {"ms": 508.123, "moves_per_row": 1725.12}
    hb = {"points": [{"had_block": b, "act_quant_us": 8.6123, "layer_us": 72.3123} for b in (16, 32, 64, 128)]}
    return sweep, overhead, prefill, qwen3, moe, prep, ceiling, flip, hb


def test_summary_is_compact():
    s = bench.summary(*_sections())
    text = json.dumps(s)
    assert len(text) < 1600, len(text)
    for key in ("sweep", "overhead", "prefill", "qwen3", "moe", "had_block", "weight_prep", "copy_ceiling"):
        assert key in s
    assert s["sweep"].count("|") == 3 and s["prefill"].count("|") == 7 and s["moe"].count("|") == 5
