"""The element-wise bounds the GPU parity tests use (tests/_gpu_util.py) catch
errors that a whole-matrix norm hides, and accept rounding-level noise on wide
and narrow matrices alike.  CPU only."""
import numpy as np

from tests._gpu_util import FRO_TOL, ROW_TOL, TILE_TOL, close_report


def _noisy(ref, rel, rng):
    return ref * (1.0 + rng.standard_normal(ref.shape) * rel)


def test_localized_errors_fail_the_row_and_tile_bounds():
    rng = np.random.default_rng(1)
    ref = rng.standard_normal((4096, 4096))
    ok = close_report(_noisy(ref, 1e-3, rng), ref)
    assert ok["fro"] <= FRO_TOL and ok["row"] <= ROW_TOL and ok["tile"] <= TILE_TOL
    bad = _noisy(ref, 1e-3, rng)
    bad[100, 640:704] *= -1.0                     # one wrong 64-column block in one row
    rep = close_report(bad, ref)
    assert rep["fro"] <= FRO_TOL                  # hidden in the whole-matrix norm ...
    assert rep["row"] > ROW_TOL and rep["tile"] > TILE_TOL   # ... but not in its row or tile
    bad = _noisy(ref, 1e-3, rng)
    bad[2000:2003, 7] = 1e3                        # a few wild outputs
    assert close_report(bad, ref)["tile"] > TILE_TOL


def test_narrow_and_tiny_matrices_accept_rounding_noise():
    rng = np.random.default_rng(2)
    for shape in [(320, 1), (320, 3), (4096, 64), (1, 11008), (16, 8)]:
        ref = rng.standard_normal(shape)
        rep = close_report(ref + rng.standard_normal(shape) * 2e-3 * np.abs(ref).mean(), ref)
        assert rep["fro"] <= FRO_TOL and rep["row"] <= ROW_TOL and rep["tile"] <= TILE_TOL, (shape, rep)
