"""The benchmark's algorithmic FLOP and byte accounting (the numerators of its
roofline figures), checked against totals worked out independently from the
shapes: per target token per block 2(4d^2 + 3dF) GEMM FLOPs plus 4(P+N)d
attention FLOPs; per cached step at full width 75.87 TFLOP (GEMM 57.17 +
attention 18.69), one block 2.38 TFLOP, the large configuration 659.7 TFLOP."""
import pytest

import bench
from qi21_synth import configs as C


@pytest.mark.parametrize("name,tflop,half_ulp", [("full", 75.87, 0.005), ("block", 2.38, 0.005),
                                                ("large", 659.7, 0.05)])
def test_step_flops(name, tflop, half_ulp):
    # the totals are given to their last printed digit: agree within half a unit of it
    assert abs(bench.step_flops(C.make_workload(name)) / 1e12 - tflop) <= half_ulp


def test_kernel_flops_add_up_to_the_step():
    w = C.make_workload("full")
    kf = bench.kernel_flops(w)
    per_layer = kf["gemm_qkv"] + kf["gemm_o"] + kf["gemm_gateup"] + kf["gemm_down"] + kf["attn"]
    img_in_out = 2 * 2 * w.shape.d_model * w.shape.latent_ch * w.n_target
    assert per_layer * w.shape.n_layers + img_in_out == bench.step_flops(w)
    # attention of one full-width layer: 4 * 4096 queries * 8704 keys * 4096 = 584.1 GFLOP
    assert kf["attn"] / 1e9 == pytest.approx(584.1, rel=1e-3)
    # GEMM share of the step: 57.17 of 75.87 TFLOP
    gemm = (kf["gemm_qkv"] + kf["gemm_o"] + kf["gemm_gateup"] + kf["gemm_down"]) * w.shape.n_layers
    assert abs(gemm / 1e12 - 57.17) <= 0.005


def test_memory_bound_bytes():
    w = C.make_workload("full")
    kb = bench.kernel_bytes(w)
    rows, d = w.n_target, w.shape.d_model
    assert kb["modln"] == rows * d * 6 == 100663296          # read fp32 h, write bf16
    assert kb["euler"] == rows * 64 * 12                      # read x and v, write x (fp32)


def test_tensor_fractions_and_clock_normalisation():
    peaks = {"bf16_tflops": 1650.0, "bf16_tflops_sustained": 1350.0, "sustained_mhz": 1200.0, "hbm_gbs": 6500.0}
    fr = bench.tensor_fracs(1080.0, peaks, 1440.0)
    assert fr["frac_sustained"] == 0.8 and fr["frac_burst"] == round(1080 / 1650, 4)
    # 1080 TF at 1440 MHz is 0.75 TF/MHz; the sustained peak is 1.125 TF/MHz
    assert fr["frac_per_clock_vs_sustained"] == round(0.75 / 1.125, 4)
    assert "frac_per_clock_vs_sustained" not in bench.tensor_fracs(1080.0, peaks, None)


def test_peak_clock_lookup():
    j = {"hbm_gbs": 6542.7, "bf16_tflops": 1650.6, "bf16_tflops_sustained": 1354.2,
         "clocks": {"bf16_sustained_sm_mhz_median": 1207, "bf16_burst_sm_mhz": 1965, "mem_mhz": 3996}}
    assert bench._find_mhz(j, True) == 1207.0
    assert bench._find_mhz(j, False) == 1965.0
    assert bench._find_mhz({"hbm_gbs": 1.0}, True) is None


def test_kernel_table_shares_and_rates():
    w = C.make_workload("full")
    prof = {"gemm_gateup": (2, 1.25), "modln": (4, 0.1), "other": (1, 0.15)}
    peaks = {"bf16_tflops": 1650.0, "bf16_tflops_sustained": 1350.0, "sustained_mhz": None, "hbm_gbs": 6500.0}
    t = bench.kernel_table(prof, bench.kernel_flops(w), bench.kernel_bytes(w), peaks, None)
    assert abs(sum(e["share"] for e in t.values()) - 1.0) < 1e-3
    assert t["gemm_gateup"]["tflops"] == round(2 * 4096 * 4096 * 24576 / 0.625e-3 / 1e12, 1)
    assert t["modln"]["gbs"] == round(4096 * 4096 * 6 / 0.025e-3 / 1e9, 1)
