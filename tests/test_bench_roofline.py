"""bench.py's roofline arithmetic on CPU: algorithmic units and the choice of
the binding bound (cache bytes at the HBM peak against contraction FLOPs at
the tensor peak)."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

PEAKS = {"hbm_gbs": 6451.8, "bf16_tflops": 1655.5, "source": "test"}


def _units(name):
    import bench
    import workloads as W
    w = W.WORKLOADS[name]
    lens = np.full(w.batch, w.seq_len, dtype=np.int64)
    return bench.algorithmic(w, lens)


def test_long_workload_units_and_hbm_bound():
    import bench
    b, f = _units("long")
    # 8 x 131,072 rows x 1152 B; 2 * 128 * (576 + 512) FLOP per visible row
    assert b == 8 * 131072 * 1152
    assert f == pytest.approx(2.0 * 128 * 8 * 131072 * 1088)
    r = bench.binding_roofline(b, f, 0.4, PEAKS, None)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(b / 0.4e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / PEAKS["hbm_gbs"])


def test_e4m3_mtp_workload_is_tensor_bound():
    import bench
    b, f = _units("fp8_mtp")
    # 580 B per e4m3 row (codes + fp32 scale); both query tokens see all but
    # the rows after them: 4095 + 4096 rows per sequence
    assert b == 128 * 4096 * 580
    assert f == pytest.approx(2.0 * 128 * 128 * (4095 + 4096) * 1088)
    r = bench.binding_roofline(b, f, 0.8, PEAKS, 123)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["traffic"] == 123
    assert r["achieved"] == pytest.approx(f / 0.8e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / PEAKS["bf16_tflops"])
    assert r["algorithmic_bytes_per_launch"] == b and r["algorithmic_flops_per_launch"] == f


def test_e4m3_operands_take_twice_the_bf16_peak():
    import bench
    b, f = _units("fp8_mtp")
    r = bench.binding_roofline(b, f, 0.3, PEAKS, None, "e4m3")
    assert r["bound"] == "tensor" and r["mma"] == "e4m3"
    assert r["peak"] == pytest.approx(2 * PEAKS["bf16_tflops"])
    assert r["frac_of_bf16_peak"] == pytest.approx(2 * r["frac"])
    assert r["frac"] == pytest.approx(f / 0.3e-3 / 1e12 / (2 * PEAKS["bf16_tflops"]))
    s = bench._decode_summary(b, f, 0.3, 0.4, PEAKS, "e4m3")
    assert s["tensor_frac_burst"] == pytest.approx(r["frac"])


def test_mma_type_of_a_step():
    import bench

    class Step:
        def __init__(self, q8, cache_dtype):
            self.q8, self.cache_dtype = q8, cache_dtype
    assert bench.mma_type(Step(True, 2)) == "e4m3"
    assert bench.mma_type(Step(False, 2)) == "f16"
    assert bench.mma_type(Step(False, 1)) == "bf16"
