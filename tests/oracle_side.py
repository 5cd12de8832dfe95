"""Comparison helper of the GPU parity tests."""
import numpy as np

from oracle.batch import OracleBatch, compact_pools  # noqa: F401


def assert_attention_close(got, ref, atol=2e-3, rtol=1e-2):
    """Elementwise |got - ref| <= atol + rtol * |ref| (fp16 output vs fp64 oracle)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    assert np.isfinite(got).all(), "non-finite outputs"
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref)
    if bad.any():
        idx = np.argwhere(bad)[:5].tolist()
        raise AssertionError("%d of %d outputs outside tolerance; first %s; max abs err %.3g" % (
            bad.sum(), bad.size, idx, err.max()))
    return float(err.max())
