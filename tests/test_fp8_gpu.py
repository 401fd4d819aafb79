"""FP8 (e4m3, one fp32 scale per cached token) cache on the GPU against the
oracle's FP8 definition, through the C ABI (``mla_decode_fp8``)."""
import numpy as np
import pytest
import torch

import decode_attention_latent_b200 as mla
import mla_inputs as mi
import oracle
from test_parity import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mla.load_library()
    return torch.device("cuda", 0)


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def run_fp8(inp, cache, dev, n_sms=None):
    q, bt, sl = inp.q.to(dev), inp.block_table.to(dev), inp.cache_seqlens.to(dev)
    n = mla.num_sms(dev) if n_sms is None else n_sms
    sched, splits = mla.decode_metadata(sl, inp.s_q, inp.H, n)
    out, lse = mla.decode_fp8(q, cache.codes.to(dev), cache.scale.to(dev), bt, sl, inp.scale, sched_meta=sched,
                              num_splits=splits, num_sms_=n)
    err = mla.get_device_error(sched)
    return out.float().cpu().numpy(), lse.cpu().numpy(), err


@pytest.mark.parametrize("seqlens,n_sms,pow2", [
    ([1, 200, 700], None, False), ([1, 200, 700], 8, True), ([64, 65, 127, 128, 129], 17, False),
    ([64 * 40 + 3, 5000], None, False), ([0, 300, 0], 7, False),
])
def test_fp8_matches_oracle(dev, orc, seqlens, n_sms, pow2):
    inp = mi.small(B=len(seqlens), s_q=1, H=16, seqlens=seqlens, seed=60)
    cache = mi.fp8_cache(inp.kv_cache.shape[0], seed=61, pow2_scales=pow2)
    g_out, g_lse, err = run_fp8(inp, cache, dev, n_sms)
    assert err == 0
    r_out, r_lse = orc.direct_fp8(inp.q, cache.codes, cache.scale, inp.block_table, inp.cache_seqlens, inp.scale)
    compare(g_out, g_lse, r_out, r_lse, what=f"fp8 {seqlens}")


def test_fp8_tail_codes_never_reach_the_result(dev, orc):
    # rows past a sequence's end hold NaN codes (0x7F) and a NaN scale
    inp = mi.small(B=2, s_q=1, H=16, seqlens=[70, 130], seed=62)
    cache = mi.fp8_cache(inp.kv_cache.shape[0], seed=63)
    for b, L in enumerate(inp.cache_seqlens.tolist()):
        last = int(inp.block_table[b, (L - 1) // 64])
        cache.codes[last, L % 64 or 64:, :] = 0x7F
        cache.scale[last, L % 64 or 64:] = float("nan")
    g_out, g_lse, err = run_fp8(inp, cache, dev)
    assert err == 0 and np.all(np.isfinite(g_out)) and np.all(np.isfinite(g_lse))
    r_out, r_lse = orc.direct_fp8(inp.q, cache.codes, cache.scale, inp.block_table, inp.cache_seqlens, inp.scale)
    compare(g_out, g_lse, r_out, r_lse, what="fp8 NaN tails")


def test_fp8_every_code_reaches_the_output_exactly(dev):
    # One visible token with scale 1: its weight is 1, so each output row is
    # the token's 512 value columns as the output MMA reads them (the codes
    # themselves, weight 1 exactly in e4m3).  The row holds every code but the
    # two NaN patterns s|1111|111, twice (subnormals and both zeros included),
    # checked against torch's float8_e4m3fn decoding.
    inp = mi.small(B=1, s_q=1, H=16, seqlens=[1], seed=68)
    cache = mi.fp8_cache(inp.kv_cache.shape[0], seed=69)
    finite = torch.tensor([c for c in range(256) if c & 0x7F != 0x7F] + [0x38, 0xB8])
    codes = torch.cat([finite, finite.flip(0), torch.full((64,), 0x38)]).to(torch.uint8)
    assert codes.numel() == 576
    blk = int(inp.block_table[0, 0])
    cache.codes[blk, 0] = codes
    cache.scale[blk, 0] = 1.0
    g_out, g_lse, err = run_fp8(inp, cache, dev)
    assert err == 0 and np.all(np.isfinite(g_lse))
    expect = codes[:512].view(torch.float8_e4m3fn).float().numpy()
    assert np.all(np.isfinite(expect))
    for h in range(16):
        np.testing.assert_array_equal(g_out[0, 0, h], expect)


@pytest.mark.parametrize("H,s_q", [(16, 1), (16, 2)])
def test_fp8_negative_and_zero_scales(dev, orc, H, s_q):
    # a token's scale may be any fp32 value: negative scales negate the row,
    # zero scales zero it (its score is 0, its value the zero vector)
    inp = mi.small(B=3, s_q=s_q, H=H, seqlens=[300, 777, 64], seed=74)
    cache = mi.fp8_cache(inp.kv_cache.shape[0], seed=75)
    g = torch.Generator().manual_seed(76)
    sign = torch.randint(0, 3, cache.scale.shape, generator=g)  # 0: negate, 1: zero, 2: keep
    cache.scale = torch.where(sign == 0, -cache.scale, torch.where(sign == 1, torch.zeros_like(cache.scale),
                                                                   cache.scale))
    g_out, g_lse, err = run_fp8(inp, cache, dev)
    assert err == 0
    r_out, r_lse = orc.direct_fp8(inp.q, cache.codes, cache.scale, inp.block_table, inp.cache_seqlens, inp.scale)
    compare(g_out, g_lse, r_out, r_lse, what=f"fp8 signed scales s_q={s_q}")


def test_fp8_paging_invariance(dev):
    # the same logical rows through an identity and a shuffled table: bitwise equal
    a = mi.small(B=2, s_q=1, H=16, seqlens=[300, 900], table="identity", seed=64)
    b = mi.small(B=2, s_q=1, H=16, seqlens=[300, 900], table="shuffled", seed=64)
    ca = mi.fp8_cache(a.kv_cache.shape[0], seed=65)
    cb = mi.Fp8Cache(codes=torch.empty_like(ca.codes), scale=torch.empty_like(ca.scale))
    for s in range(2):
        for p in range((int(a.cache_seqlens[s]) + 63) // 64):
            cb.codes[int(b.block_table[s, p])] = ca.codes[int(a.block_table[s, p])]
            cb.scale[int(b.block_table[s, p])] = ca.scale[int(a.block_table[s, p])]
    oa = run_fp8(a, ca, dev, 8)
    ob = run_fp8(b, cb, dev, 8)
    assert np.array_equal(oa[0], ob[0]) and np.array_equal(oa[1], ob[1])


@pytest.mark.parametrize("H,s_q,seqlens,n_sms", [
    (32, 1, [1, 200, 700], None), (32, 1, [64, 65, 127, 128, 129], 17),
    (16, 2, [2, 200, 700], None), (16, 2, [64, 65, 127, 128, 129], 17), (16, 2, [64 * 40 + 3, 5000], 11),
])
def test_fp8_32_query_columns(dev, orc, H, s_q, seqlens, n_sms):
    # 32 query columns: 32 heads, or 16 heads at two query positions (causal)
    inp = mi.small(B=len(seqlens), s_q=s_q, H=H, seqlens=seqlens, seed=70)
    cache = mi.fp8_cache(inp.kv_cache.shape[0], seed=71)
    g_out, g_lse, err = run_fp8(inp, cache, dev, n_sms)
    assert err == 0
    r_out, r_lse = orc.direct_fp8(inp.q, cache.codes, cache.scale, inp.block_table, inp.cache_seqlens, inp.scale)
    compare(g_out, g_lse, r_out, r_lse, what=f"fp8 H={H} s_q={s_q} {seqlens}")


def test_fp8_last_token_seen_by_the_second_query_position(dev, orc):
    # s_q = 2: the last cached token is visible to query position 1 only; NaN
    # codes and scales past the sequence end must still not reach the result
    inp = mi.small(B=2, s_q=2, H=16, seqlens=[70, 129], seed=72)
    cache = mi.fp8_cache(inp.kv_cache.shape[0], seed=73)
    for b, L in enumerate(inp.cache_seqlens.tolist()):
        last = int(inp.block_table[b, (L - 1) // 64])
        cache.codes[last, L % 64 or 64:, :] = 0x7F
        cache.scale[last, L % 64 or 64:] = float("nan")
        cache.scale[last, (L - 1) % 64] = 4.0  # the last token weighs in visibly for position 1
    g_out, g_lse, err = run_fp8(inp, cache, dev)
    assert err == 0 and np.all(np.isfinite(g_out)) and np.all(np.isfinite(g_lse))
    r_out, r_lse = orc.direct_fp8(inp.q, cache.codes, cache.scale, inp.block_table, inp.cache_seqlens, inp.scale)
    compare(g_out, g_lse, r_out, r_lse, what="fp8 s_q=2 last token")


@pytest.mark.parametrize("name", ["b8_h16_l64k", "b32_sq2_h16_l16k_outliers"])
def test_fp8_full_size_workload(dev, orc, name):
    # the launch configuration `bench.py --fp8` times (metadata, attention and
    # combine over every SM), on its inputs at full size; every sequence checked
    inp = mi.make_inputs(mi.WORKLOADS[name], seed=0)
    nb = inp.kv_cache.shape[0]
    inp.kv_cache = None
    cache = mi.fp8_cache(nb, seed=1)
    g_out, g_lse, err = run_fp8(inp, cache, dev)
    assert err == 0
    r_out, r_lse = orc.direct_fp8(inp.q, cache.codes, cache.scale, inp.block_table, inp.cache_seqlens, inp.scale)
    compare(g_out, g_lse, r_out, r_lse, what=f"fp8 {name}")


@pytest.mark.parametrize("H,s_q", [(16, 1), (16, 2)])
def test_fp8_bad_block_table_sets_error_word(dev, orc, H, s_q):
    # an entry naming no block of the cache: both loads of its tile read
    # block 0 instead, the error word says so, and the other sequence is exact
    inp = mi.small(B=2, s_q=s_q, H=H, seqlens=[300, 200], seed=74)
    cache = mi.fp8_cache(inp.kv_cache.shape[0], seed=75)
    good = inp.block_table[0:1].clone()
    inp.block_table[1, 2] = inp.kv_cache.shape[0] + 5
    g_out, g_lse, err = run_fp8(inp, cache, dev)
    assert err & mla.DEVERR_BLOCK_TABLE
    r_out, r_lse = orc.direct_fp8(inp.q[0:1], cache.codes, cache.scale, good, inp.cache_seqlens[0:1], inp.scale)
    compare(g_out[0:1], g_lse[0:1], r_out, r_lse, what=f"fp8 bad page, other sequence (s_q={s_q})")


@pytest.mark.parametrize("H,s_q", [(64, 1), (32, 2), (16, 4), (128, 1)])
def test_fp8_unsupported_shape_is_refused(dev, H, s_q):
    inp = mi.small(B=1, s_q=s_q, H=H, seqlens=[100], seed=66)
    cache = mi.fp8_cache(inp.kv_cache.shape[0], seed=67)
    with pytest.raises(mla.MLAError):
        mla.decode_fp8(inp.q.to(dev), cache.codes.to(dev), cache.scale.to(dev), inp.block_table.to(dev),
                       inp.cache_seqlens.to(dev), inp.scale)
