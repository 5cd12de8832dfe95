"""Comparison helpers of the GPU parity tests."""
import numpy as np

from oracle.batch import OracleBatch, compact_pools  # noqa: F401

#: (config, outputs compared, max abs error, max rel error over |ref| > 1e-3) of every
#: attention comparison recorded in this session; conftest prints them at the end
ERRORS = []


def assert_attention_close(got, ref, atol=2e-3, rtol=1e-2, record=None, literal=False):
    """Elementwise |got - ref| <= atol + rtol * |ref| (fp16 output vs fp64 oracle).

    record: a config name under which the max abs / rel errors are kept for the session
    summary.  literal: also require max |got - ref| <= atol (the target's "max abs error
    2e-3" read literally, for the full-size configs whose outputs are small)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    assert np.isfinite(got).all(), "non-finite outputs"
    err = np.abs(got - ref)
    big = np.abs(ref) > 1e-3
    rel = float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    if record is not None:
        ERRORS.append((record, int(err.size), float(err.max()), rel))
    bad = err > atol + rtol * np.abs(ref)
    if bad.any():
        idx = np.argwhere(bad)[:5].tolist()
        raise AssertionError("%d of %d outputs outside tolerance; first %s; max abs err %.3g" % (
            bad.sum(), bad.size, idx, err.max()))
    if literal:
        assert err.max() <= atol, "max abs error %.3g above %.3g" % (err.max(), atol)
    return float(err.max())
