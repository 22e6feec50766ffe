"""Host-side logic of bench.py that needs no GPU: which kernel the bench line's roofline
reports, and where its DRAM traffic comes from."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_dominant_kernel_sums_both_projections():
    sys.path.insert(0, ROOT)
    import bench
    names = ["quant_int4_up", "quant_int4_down", "gemm_w8a8", "gemv_w4a16_b1_up", "gemv_w4a16_b1_down"]
    # the single longest launch is the W8A8 GEMM, but the INT4 quantizer's two launches together
    # take more of the step; its first launch is reported, whichever of the two is longer
    us = {"quant_int4_up": 150.0, "quant_int4_down": 151.0, "gemm_w8a8": 170.0,
          "gemv_w4a16_b1_up": 33.0, "gemv_w4a16_b1_down": 34.0}
    assert bench.dominant_kernel(names, us) == "quant_int4_up"
    us["gemm_w8a8"] = 400.0
    assert bench.dominant_kernel(names, us) == "gemm_w8a8"
    assert bench.load_traffic("quant_int4_up") > 0


def test_reference_arm_line_has_the_contract_keys():
    # The reference arm times the CPU oracle on a bounded sample and prints one JSON line with
    # the same metric, unit and config as the GPU arm.
    import contextlib
    import io
    import json
    sys.path.insert(0, ROOT)
    import bench
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--cpu-seconds", "1"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "GB/s"
    assert line["value"] > 0 and line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["config"] == bench.arm_config(1) and "workload" in line["config"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == "GB/s"
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
