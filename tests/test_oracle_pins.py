"""The oracle against its pins (CPU only)."""
import json
import os

import pytest

import oracle
from tests import pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def orc():
    return oracle.oracle()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_distinct_offsets_match_page(orc):
    with open(os.path.join(GOLDEN, "rpb_table_entries.json")) as f:
        g = json.load(f)
    pins.pin_distinct_offsets(orc, M=g["M"], expected=g["entries_per_head"])


def test_units_match_full_map(orc):
    """fwd_units (sampled units, window order) agrees with fwd (whole map)."""
    import numpy as np
    q, k, v = pins._maps((2, 8, 8, 3, 8), "bf16", "units-vs-map")
    M, s = 4, 2
    full = orc.fwd(q, k, v, M=M, shift=s)
    units = [0, 5, 7, 23]
    got = orc.fwd_units(q, k, v, units, M=M, shift=s)
    nWy, nWx, heads = 2, 2, 3
    for n, u in enumerate(units):
        h = u % heads
        w = u // heads
        wx, wy, b = w % nWx, (w // nWx) % nWy, w // (nWx * nWy)
        for p in range(M * M):
            y, x = orc.token_origin(8, 8, M, s, wy, wx, p)
            assert np.array_equal(got[n, p], full[b, y, x, h])


def test_rejects_bad_problems(orc):
    q, k, v = pins._maps((1, 8, 8, 1, 8), "fp32", "reject")
    with pytest.raises(ValueError):
        orc.fwd(q, k, v, M=0)            # windows need M >= 1
    with pytest.raises(ValueError):
        orc.fwd(q, k, v, M=4, shift=4)   # shift must be < M
