"""The library's spatial token order (a host function, no GPU needed) against
the oracle's, on the VGGT geometry and on small hand-checkable grids."""
import ctypes

import numpy as np
import pytest

import oracle


def _order(lib, views, grid, specials, wr, wc):
    n = views * (specials + grid * grid)
    order = (ctypes.c_int32 * n)()
    inv = (ctypes.c_int32 * n)()
    st = lib.zb_spatial_order(views, grid, specials, wr, wc, order, inv)
    return st, np.frombuffer(order, dtype=np.int32).copy(), np.frombuffer(inv, dtype=np.int32).copy()


@pytest.mark.parametrize("geom", [(32, 37, 5, 8, 16), (3, 37, 5, 16, 8), (2, 5, 1, 2, 3), (4, 9, 0, 4, 4),
                                  (1, 37, 5, 37, 37)])
def test_spatial_order_matches_oracle(geom):
    from linear_hybrid_attention_b200 import _lib
    lib = _lib.load()
    st, order, inv = _order(lib, *geom)
    assert st == 0
    want = oracle.spatial_order(geom[0], grid=geom[1], specials=geom[2], win_rows=geom[3], win_cols=geom[4])
    np.testing.assert_array_equal(order, want)
    np.testing.assert_array_equal(inv, oracle.inverse_order(want))


def test_spatial_order_rejects_bad_geometry():
    from linear_hybrid_attention_b200 import _lib
    lib = _lib.load()
    assert lib.zb_spatial_order(0, 37, 5, 8, 16, None, None) == 2      # ZB_ERR_SHAPE
    assert lib.zb_spatial_order(1, 37, 5, 0, 16, None, None) == 2
    assert lib.zb_spatial_order(1, 37, 5, 8, 16, None, None) == 1      # ZB_ERR_NULL
