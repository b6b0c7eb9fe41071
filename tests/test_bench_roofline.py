"""bench.py's per-kernel roofline entries on CPU: a tensor-bound kernel carries
its fraction of the measured FP8 figure and of both of the library's own
probe figures (Gaussian operand codes, the denominator of fp8_frac_own, and
low-toggle codes beside it); an HBM-bound one carries no FP8 fractions; and
the stored ncu traffic figures name kernels whose sources can be hashed."""

import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


OWN = {"fp8_dense_tflops": 4000.0, "fp8_dense_tflops_low_toggle": 5000.0,
       "hbm_copy_gbs": 6000.0}


def test_tensor_bound_entry_carries_both_own_fractions():
    b = _bench()
    k = b.Kern("gemm_rope_kv", "tensor", algo_bytes=1e9, flops=2e12)
    e = b._kern_entry(1.0, k, 6500.0, 3200.0, OWN)   # 1 ms per launch
    assert e["TFLOP_s"] == pytest.approx(2000.0)
    assert e["fp8_frac"] == pytest.approx(2000.0 / 3200.0, abs=1e-4)
    assert e["fp8_frac_own"] == pytest.approx(0.5, abs=1e-4)
    assert e["fp8_frac_own_low_toggle"] == pytest.approx(0.4, abs=1e-4)
    assert e["GB_s"] == pytest.approx(1000.0)
    assert e["hbm_frac_own"] == pytest.approx(1000.0 / 6000.0, abs=1e-4)


def test_hbm_bound_entry_has_no_fp8_fractions():
    b = _bench()
    k = b.Kern("producer", "hbm", algo_bytes=3.25e9)
    e = b._kern_entry(1.0, k, 6500.0, 3200.0, OWN)
    assert e["hbm_frac"] == pytest.approx(0.5, abs=1e-4)
    assert "TFLOP_s" not in e and "fp8_frac_own" not in e


def test_stored_traffic_names_hashable_sources():
    b = _bench()
    # every stored figure names a kernel whose sources exist and hash to a
    # 16-hex-digit digest (a figure whose digest no longer matches is
    # reported as null, not used)
    for (_, kern), (traffic, digest) in b.NCU_TRAFFIC.items():
        assert traffic > 0
        h = b._src_hash(kern)
        assert len(h) == 16 and int(h, 16) >= 0
        assert len(digest) == 16
