"""The fp64 oracle against its pins (CPU only)."""
import numpy as np
import pytest
import torch

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


def test_fp8_cache_recipe():
    # seeded, free of NaN codes (exponent field <= 14), magnitudes around 1
    a = mi.fp8_cache(3, seed=9)
    b = mi.fp8_cache(3, seed=9)
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scale, b.scale)
    assert a.codes.dtype == torch.uint8 and a.codes.shape == (3, 64, 576) and a.scale.shape == (3, 64)
    expo = (a.codes.to(torch.int64) >> 3) & 15
    assert int(expo.max()) <= 14
    vals = a.codes.view(torch.float8_e4m3fn).to(torch.float64)
    assert torch.isfinite(vals).all() and 0.3 < float(vals.abs().median()) < 3.0
    assert float(a.scale.min()) >= 0.05 and float(a.scale.max()) < 0.3
    p2 = mi.fp8_cache(2, seed=9, pow2_scales=True).scale
    assert torch.equal(p2, torch.exp2(torch.round(torch.log2(p2))))


def test_fp8_oracle_rejects_bad_block(orc):
    inp = mi.small(B=1, s_q=1, H=1, seqlens=[70], seed=5)
    c = mi.fp8_cache(inp.kv_cache.shape[0], seed=6)
    inp.block_table[0, 1] = inp.kv_cache.shape[0]
    with pytest.raises(ValueError):
        orc.direct_fp8(inp.q, c.codes, c.scale, inp.block_table, inp.cache_seqlens, inp.scale)
