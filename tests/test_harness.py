"""The parity measures of the GPU tests, checked on the CPU (no GPU needed)."""
import numpy as np

from edge_aware_graph_b200 import inputs as I

from harness import increment_err, rel_err


def test_increment_measure_ignores_storage_rounding_only():
    rng = np.random.default_rng(0)
    base = I.to_storage(rng.standard_normal((64, 64)) * 3.0, "bf16").astype(np.float64)
    inc = rng.standard_normal((64, 64)) * 0.05
    ref = base + inc
    stored = I.to_storage(ref.astype(np.float32), "bf16")           # round to nearest even
    # rounding the exact output to the storage dtype is not an error of the increment
    assert increment_err(stored, base, ref, "bf16") == 0.0
    # while measured on the output's scale the same rounding looks small ...
    assert rel_err(stored, ref) < 5e-3
    # ... a wrong increment of 3% of the increment scale on one pair is caught
    bad = stored.astype(np.float64).copy()
    bad[5, 7] += 0.03 * np.abs(inc).max() + 0.1
    bad = I.to_storage(bad.astype(np.float32), "bf16")
    assert increment_err(bad, base, ref, "bf16") > 2e-2
    # and so is a dropped increment on the small-update pairs
    dropped = np.where(np.abs(inc) < 0.5 * np.abs(inc).max(), base, stored)
    assert increment_err(dropped, base, ref, "bf16") > 0.4


def test_increment_measure_fp32():
    rng = np.random.default_rng(1)
    base = rng.standard_normal(1000).astype(np.float32).astype(np.float64)
    ref = base + 1e-3 * rng.standard_normal(1000)
    assert increment_err(ref.astype(np.float32), base, ref, "fp32") == 0.0
    assert increment_err((ref + 1e-5).astype(np.float32), base, ref, "fp32") > 1e-3
