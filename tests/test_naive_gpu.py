"""The non-absorbed form on the GPU (mla_decode_naive, through the C ABI)
against the oracle's definition of it (mla_oracle_naive, fp64), with the
tolerances of test_parity.py: per tile the keys and values are decompressed
from the latent rows by the per-head up-projections on the tensor cores."""
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


def run_naive(base, nv, dev, n_sms=None):
    out, lse, err = mla.decode_naive(nv.q.to(dev), base.kv_cache.to(dev), nv.w_uk.to(dev), nv.w_uv.to(dev),
                                     base.block_table.to(dev), base.cache_seqlens.to(dev), base.scale,
                                     num_sms_=n_sms)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), int(err.item())


@pytest.mark.parametrize("s_q,H,lens,n_sms", [
    (1, 16, [1, 63, 64, 65, 127, 128, 129, 1000], None),
    (2, 16, [1, 2, 64, 65, 130, 700], None),
    (1, 4, [5000, 3, 0, 2600], 8),
    (2, 2, [4096 + 17], 148),
    (1, 128, [300, 1200], None),
])
def test_naive_matches_oracle(dev, orc, s_q, H, lens, n_sms):
    base = mi.small(B=len(lens), s_q=s_q, H=H, seqlens=lens, seed=400 + H + s_q, tail_fill=float("nan"))
    nv = mi.naive_inputs(len(lens), s_q, H, seed=401 + H)
    g_out, g_lse, err = run_naive(base, nv, dev, n_sms)
    assert err == 0
    r_out, r_lse = orc.naive(nv.q, base.kv_cache, nv.w_uk, nv.w_uv, base.block_table, base.cache_seqlens, base.scale)
    compare(g_out, g_lse, r_out, r_lse, what=f"naive s_q={s_q} H={H}")


def test_naive_full_size_workload(dev, orc):
    # the launch configuration `bench.py --naive` times: the 64K-context,
    # 16-head workload at full size over every SM; the oracle checks two
    # whole sequences (its per-token decompression makes all eight slow)
    w = mi.WORKLOADS["b8_h16_l64k"]
    base = mi.make_inputs(w, seed=0)
    nv = mi.naive_inputs(w.B, w.s_q, w.H, seed=1)
    g_out, g_lse, err = run_naive(base, nv, dev)
    assert err == 0
    seqs = [0, 5]
    r_out, r_lse = orc.naive(nv.q, base.kv_cache, nv.w_uk, nv.w_uv, base.block_table, base.cache_seqlens,
                             base.scale, seqs=seqs)
    compare(g_out, g_lse, r_out, r_lse, seqs=seqs, what="naive b8_h16_l64k")


def test_naive_page_table_invariance(dev):
    """The same logical rows through an identity and a shuffled table give
    bitwise equal results (integer page indexing is exact)."""
    lens = [3000, 640, 129]
    ident = mi.small(B=3, s_q=1, H=8, seqlens=lens, table="identity", seed=410)
    shuf = mi.small(B=3, s_q=1, H=8, seqlens=lens, table="shuffled", seed=410)
    kv = torch.empty_like(ident.kv_cache)
    for b, L in enumerate(lens):
        for p in range(mi.pages_for(L)):
            kv[int(shuf.block_table[b, p])] = ident.kv_cache[int(ident.block_table[b, p])]
    shuf.kv_cache = kv
    nv = mi.naive_inputs(3, 1, 8, seed=411)
    a = run_naive(ident, nv, dev)
    b = run_naive(shuf, nv, dev)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_naive_bad_page_sets_error_word(dev):
    base = mi.small(B=2, s_q=1, H=2, seqlens=[300, 200], seed=412)
    base.block_table[1, 2] = base.kv_cache.shape[0] + 5
    nv = mi.naive_inputs(2, 1, 2, seed=413)
    _, _, err = run_naive(base, nv, dev)
    assert err & mla.DEVERR_BLOCK_TABLE
