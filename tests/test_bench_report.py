"""The bench line's stage report and roofline (host arithmetic only, no GPU): which kernel is
the dominant one for each workload kind, which bound applies, and that every fraction is the
stated bytes or flops over the stage time over the measured peak."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402

PEAKS = {"hbm_gbs": 6543.4, "bf16_tflops": 1617.4}


def _mean(ms):
    up, down = ms.get("up_gate", 0.0), ms.get("down", 0.0)
    return {"permute": ms["permute"], "up_gate": up, "down": down, "ffn": up + down,
            "combine": ms["combine"]}


def _report(wname, ms, **kw):
    w = synth.WORKLOADS[wname]
    return w, bench.stage_report(w, w.E, w.K, None, _mean(ms), PEAKS, "measured", **kw)


def test_full_size_layer_is_hbm_bound_on_the_swiglu_pass():
    w, (stages, roof) = _report("large", {"permute": 0.3, "up_gate": 4.0, "down": 2.5,
                                          "combine": 0.25})
    wm = bench.work_model(w)
    assert roof["kernel"].startswith("grouped_ffn_kernel<0>")
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert roof["achieved"] == pytest.approx(wm["up_gate_bytes"] / 4.0e-3 / 1e9)
    assert roof["frac"] == pytest.approx(roof["achieved"] / PEAKS["hbm_gbs"])
    # both fractions of every GEMM pass, HBM fractions of permute and combine
    for key in ("up_gate", "down", "grouped_ffn"):
        assert 0 < stages[key]["frac_tensor"] < 1 and 0 < stages[key]["frac_hbm"] < 1.2
    assert stages["down"]["GB/s"] == pytest.approx(wm["down_bytes"] / 2.5e-3 / 1e9)
    assert stages["grouped_ffn"]["TFLOP/s"] == pytest.approx(
        (wm["up_gate_flops"] + wm["down_flops"]) / 6.5e-3 / 1e12)
    for key in ("permute", "combine"):
        assert stages[key]["frac_hbm"] == pytest.approx(stages[key]["GB/s"] / PEAKS["hbm_gbs"])
    assert stages["permute"]["GB/s"] == pytest.approx(wm["permute_bytes"] / 0.3e-3 / 1e9)
    assert roof["traffic"] is None or roof["traffic"] > 0


def test_medium_layer_is_tensor_bound():
    w, (stages, roof) = _report("medium", {"permute": 0.03, "up_gate": 0.235, "down": 0.13,
                                           "combine": 0.033})
    wm = bench.work_model(w)
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["peak"] == PEAKS["bf16_tflops"]
    assert roof["achieved"] == pytest.approx(wm["up_gate_flops"] / 0.235e-3 / 1e12)
    assert stages["up_gate"]["frac_tensor"] == pytest.approx(roof["frac"])


def test_identity_expert_workload_reports_the_permutation():
    w, (stages, roof) = _report("permute_combine_S1024_mv0", {"permute": 0.03, "combine": 0.04})
    assert roof["kernel"].startswith("moe_permute") and roof["bound"] == "hbm"
    assert "up_gate" not in stages and roof["traffic"] is None
    assert roof["achieved"] == pytest.approx(bench.work_model(w)["permute_bytes"] / 0.03e-3 / 1e9)


def test_mxfp8_peaks_and_bounds():
    _, (_, roof_m) = _report("medium", {"permute": 0.03, "up_gate": 0.17, "down": 0.09,
                                        "combine": 0.033}, mx=True)
    assert roof_m["kernel"].startswith("grouped_ffn_mx_kernel")
    assert roof_m["bound"] == "tensor" and roof_m["peak"] == 2 * PEAKS["bf16_tflops"]
    w, (stages, roof_l) = _report("large", {"permute": 0.2, "up_gate": 2.6, "down": 1.8,
                                            "combine": 0.23}, mx=True)
    assert roof_l["bound"] == "hbm"
    assert roof_l["achieved"] == pytest.approx(bench.work_model(w)["up_gate_mx_bytes"] / 2.6e-3 / 1e9)
    assert stages["up_gate"]["frac_tensor"] == pytest.approx(
        stages["up_gate"]["TFLOP/s"] / (2 * PEAKS["bf16_tflops"]))


def test_zero_copy_and_shared_experts():
    w, (stages, roof) = _report("medium", {"permute": 0.014, "up_gate": 0.256, "down": 0.13,
                                           "combine": 0.033}, zero_copy=True)
    wm = bench.work_model(w)
    assert roof["kernel"].startswith("grouped_ffn_kernel<3>")
    # metadata-only permutation: its bytes exclude the row copy
    assert stages["permute"]["GB/s"] == pytest.approx(wm["permute_meta_bytes"] / 0.014e-3 / 1e9)
    assert stages["up_gate"]["GB/s"] == pytest.approx(wm["up_gate_zc_bytes"] / 0.256e-3 / 1e9)
    _, (_, roof_s) = _report("medium", {"permute": 0.03, "up_gate": 0.26, "down": 0.15,
                                        "combine": 0.04}, shared=True)
    assert roof_s["traffic"] is None  # a capture holds for its own launch shape only
