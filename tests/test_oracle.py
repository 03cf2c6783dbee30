"""The fp64 oracle against its pins (CPU only)."""
import numpy as np
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_threads_do_not_change_results(orc):
    c = pins.rand_case(31, 2, 8, 4, 40, 5, 32, mask_p=0.1)
    o1, l1 = pins.run(orc, c, nthreads=1)
    o4, l4 = pins.run(orc, c, nthreads=4)
    assert np.array_equal(o1, o4) and np.array_equal(l1, l4)


def test_bad_shapes_rejected(orc):
    c = pins.rand_case(32, 1, 4, 2, 4, 2, 8)
    for bad in (dict(Hq=3), dict(S=0), dict(Hkv=0)):
        cc = dict(c, **bad)
        with pytest.raises(ValueError):
            pins.run(orc, cc)


def test_row_range_selects_rows(orc):
    c = pins.rand_case(33, 2, 4, 2, 9, 3, 8, mask_p=0.2)
    o_full, l_full = pins.run(orc, c)
    o_part, l_part = pins.run(orc, c, row_range=(5, 17))
    flat_o, flat_l = o_part.reshape(-1, 8), l_part.reshape(-1)
    assert np.array_equal(flat_o[5:17], o_full.reshape(-1, 8)[5:17])
    assert np.array_equal(flat_l[5:17], l_full.reshape(-1)[5:17])
    assert not flat_o[:5].any() and not flat_o[17:].any()
