"""The fp64 oracle against facts other than itself (CPU only)."""
import pytest

import oracle
from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle)


def test_row_subset_matches_full_scan():
    """Computing a subset of rows gives the same values as the full scan."""
    import numpy as np
    g = np.random.default_rng(5)
    batch, dim, N, L = 2, 5, 3, 17
    kw = dict(u=g.normal(size=(batch, dim, L)).astype(np.float32),
              delta=g.normal(size=(batch, dim, L)).astype(np.float32),
              B=g.normal(size=(batch, N, L)).astype(np.float32),
              C=g.normal(size=(batch, N, L)).astype(np.float32),
              A=-np.exp(g.normal(size=(dim, N))).astype(np.float32))
    y, h = oracle.scan(**kw)
    rows = [7, 0, 9, 3]
    ys, hs = oracle.scan(**kw, rows=rows)
    assert np.array_equal(ys, y.reshape(batch * dim, L)[rows])
    assert np.array_equal(hs, h.reshape(batch * dim, N)[rows])


def test_rejects_bad_rows():
    import numpy as np
    z = np.zeros((1, 2, 3), np.float32)
    with pytest.raises(ValueError):
        oracle.scan(u=z, delta=z, B=np.zeros((1, 1, 3), np.float32),
                    C=np.zeros((1, 1, 3), np.float32), A=np.zeros((2, 1), np.float32), rows=[2])
