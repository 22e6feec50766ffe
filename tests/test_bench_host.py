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
