"""The fp64 oracle against its pins (CPU only)."""
import numpy as np
import pytest

import mla_inputs as mi
import oracle
from oracle_pins import ALL_PINS


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_bad_block_table_is_rejected(orc):
    inp = mi.small(B=1, s_q=1, H=1, seqlens=[70], seed=3)
    inp.block_table[0, 1] = inp.kv_cache.shape[0]  # one past the last block
    with pytest.raises(ValueError):
        orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)


def test_sequence_subset_leaves_other_rows_untouched(orc):
    inp = mi.small(B=3, s_q=1, H=2, seqlens=[10, 20, 30], seed=4)
    full = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    part = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale, seqs=[2, 0])
    assert np.array_equal(part[0][[0, 2]], full[0][[0, 2]])
    assert np.isnan(part[0][1]).all() and np.isnan(part[1][1]).all()
