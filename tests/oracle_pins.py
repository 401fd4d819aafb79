"""Checks that pin the fp64 oracle to facts outside itself.

Each pin takes an ``oracle.Oracle`` and raises AssertionError on a mismatch.
They compare against closed forms, library routines (torch's
scaled_dot_product_attention and logsumexp in float64) and invariants that
the definition implies -- never against a retyped copy of the oracle's own
formula.  ``test_oracle.py`` runs them on the oracle;
``test_oracle_mutants.py`` runs them on copies of the oracle with a planted
mistake and requires that some pin fails for every mistake.

Source of the definition: the FlashMLA-ETAP explainer (gist.science),
technical summary, "Methodology / core mechanism" (softmax(Q K^T) V and its
transposed form), and "FlashMLA: compressing the KV cache" (jsqmd.com),
"compute flow", step 4 (online softmax).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import mla_inputs as mi

REL = 1e-12


def _bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def _close(a, b, rel=REL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    fin = ~both_inf
    assert np.all(np.isfinite(a[fin])) and np.all(np.isfinite(b[fin])), what
    scale = max(1.0, float(np.max(np.abs(b[fin])))) if fin.any() else 1.0
    err = float(np.max(np.abs(a[fin] - b[fin]))) if fin.any() else 0.0
    assert err <= rel * scale, f"{what}: max abs err {err:.3e} > {rel * scale:.3e}"


def _rows_of(inp: mi.Inputs, b: int, n: int) -> np.ndarray:
    """Logical cache rows 0..n-1 of sequence b, gathered through the table."""
    kv = _bf16_to_f64(inp.kv_cache)
    rows = [kv[int(inp.block_table[b, j // 64]), j % 64] for j in range(n)]
    return np.stack(rows) if rows else np.zeros((0, 576))


# ---------------------------------------------------------------------------
def pin_single_token(orc):
    """A one-token context returns that token's value row exactly (its single
    weight is exp(0) = 1), and lse is the scaled score of that token."""
    inp = mi.small(B=3, s_q=1, H=4, seqlens=[1, 1, 1], seed=11)
    out, lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    q = _bf16_to_f64(inp.q)
    for b in range(3):
        row = _rows_of(inp, b, 1)[0]
        for h in range(4):
            assert np.array_equal(out[b, 0, h], row[:512]), "single token: out != v row"
            _close(lse[b, 0, h], inp.scale * float(np.dot(q[b, 0, h], row)), what="single token lse")


def pin_equal_scores_mean_of_values(orc):
    """When every key scores the same (query zero on the latent part, keys
    sharing one rope part), the result is the plain mean of the value rows
    and lse = s + ln(L)."""
    L = 77
    inp = mi.small(B=1, s_q=1, H=2, seqlens=[L], seed=12)
    inp.q[..., :512] = 0
    shared_rope = inp.kv_cache[int(inp.block_table[0, 0]), 0, 512:].clone()
    for j in range(L):
        inp.kv_cache[int(inp.block_table[0, j // 64]), j % 64, 512:] = shared_rope
    out, lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    rows = _rows_of(inp, 0, L)
    q = _bf16_to_f64(inp.q)
    for h in range(2):
        _close(out[0, 0, h], rows[:, :512].mean(axis=0), what="equal scores: mean of V")
        s = inp.scale * float(np.dot(q[0, 0, h], rows[0]))
        _close(lse[0, 0, h], s + math.log(L), what="equal scores: lse")


def pin_zero_scale(orc):
    """scale = 0 makes every weight equal: mean of V and lse = ln(n)."""
    inp = mi.small(B=2, s_q=2, H=2, seqlens=[5, 130], scale=0.0, seed=13)
    out, lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, 0.0)
    for b, L in enumerate([5, 130]):
        for i in range(2):
            n = L - 1 + i
            rows = _rows_of(inp, b, n)
            for h in range(2):
                _close(out[b, i, h], rows[:, :512].mean(axis=0), what="zero scale: mean")
                _close(lse[b, i, h], math.log(n), what="zero scale: lse = ln n")


def pin_weights_sum_to_one(orc):
    """Value rows that are all ones give all ones: the weights sum to 1."""
    inp = mi.small(B=2, s_q=1, H=3, seqlens=[200, 64], seed=14)
    inp.kv_cache[..., :512] = 1.0
    out, lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    assert np.all(np.abs(out - 1.0) <= 1e-14), "constant V: weights do not sum to 1"


def pin_two_token_closed_form(orc):
    """Two tokens with small-integer entries: the scores are exact, and the
    result is the closed form softmax of two numbers."""
    inp = mi.small(B=1, s_q=1, H=1, seqlens=[2], table="identity", scale=0.5, seed=15)
    inp.q.zero_()
    inp.kv_cache.zero_()
    inp.q[0, 0, 0, 3] = 2.0       # latent dim 3
    inp.q[0, 0, 0, 540] = -1.0    # rope dim 540
    inp.kv_cache[0, 0, 3] = 1.0
    inp.kv_cache[0, 0, 540] = 3.0
    inp.kv_cache[0, 0, 7] = 5.0
    inp.kv_cache[0, 1, 3] = 4.0
    inp.kv_cache[0, 1, 540] = -2.0
    inp.kv_cache[0, 1, 7] = -1.0
    s0 = 0.5 * (2 * 1 + (-1) * 3)    # -0.5
    s1 = 0.5 * (2 * 4 + (-1) * (-2))  # 5.0
    e0, e1 = math.exp(s0), math.exp(s1)
    want = np.zeros(512)
    want[3] = (e0 * 1 + e1 * 4) / (e0 + e1)
    want[7] = (e0 * 5 + e1 * -1) / (e0 + e1)
    out, lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, 0.5)
    _close(out[0, 0, 0], want, what="two tokens: out")
    _close(lse[0, 0, 0], math.log(e0 + e1), what="two tokens: lse")


def pin_torch_sdpa(orc):
    """Against torch's scaled_dot_product_attention (float64, CPU) on the
    gathered rows, query i seeing the first seqlen - s_q + 1 + i rows, with
    torch.logsumexp for the lse.  Shuffled pages, ragged lengths, s_q = 2."""
    lens = [1, 63, 64, 65, 130, 300]
    inp = mi.small(B=len(lens), s_q=2, H=3, seqlens=lens, seed=16)
    out, lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    q = torch.from_numpy(_bf16_to_f64(inp.q))
    for b, L in enumerate(lens):
        rows = torch.from_numpy(_rows_of(inp, b, L))
        for i in range(2):
            n = max(0, L - 1 + i)
            if n == 0:
                assert np.all(out[b, i] == 0) and np.all(np.isneginf(lse[b, i])), "empty context"
                continue
            k = rows[:n].unsqueeze(0)                 # [1, n, 576]
            v = rows[:n, :512].unsqueeze(0)           # [1, n, 512]
            qq = q[b, i].unsqueeze(1)                 # [H, 1, 576]
            ref = torch.nn.functional.scaled_dot_product_attention(
                qq, k.expand(3, n, 576), v.expand(3, n, 512), scale=inp.scale)
            _close(out[b, i], ref[:, 0].numpy(), what=f"sdpa b={b} i={i}")
            scores = inp.scale * (qq[:, 0] @ rows[:n].T)
            _close(lse[b, i], torch.logsumexp(scores, dim=-1).numpy(), what=f"lse b={b} i={i}")


def pin_torch_sdpa_four_queries(orc):
    """As pin_torch_sdpa with s_q = 4: query i sees the first seqlen - 3 + i
    rows, none when that is <= 0 (lengths 1 and 2 leave some queries empty)."""
    lens = [1, 2, 3, 4, 70, 129]
    inp = mi.small(B=len(lens), s_q=4, H=2, seqlens=lens, seed=27)
    out, lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    q = torch.from_numpy(_bf16_to_f64(inp.q))
    for b, L in enumerate(lens):
        rows = torch.from_numpy(_rows_of(inp, b, L))
        for i in range(4):
            n = max(0, L - 3 + i)
            if n == 0:
                assert np.all(out[b, i] == 0) and np.all(np.isneginf(lse[b, i])), "empty context"
                continue
            k = rows[:n].unsqueeze(0)
            v = rows[:n, :512].unsqueeze(0)
            qq = q[b, i].unsqueeze(1)
            ref = torch.nn.functional.scaled_dot_product_attention(
                qq, k.expand(2, n, 576), v.expand(2, n, 512), scale=inp.scale)
            _close(out[b, i], ref[:, 0].numpy(), what=f"sdpa4 b={b} i={i}")
            scores = inp.scale * (qq[:, 0] @ rows[:n].T)
            _close(lse[b, i], torch.logsumexp(scores, dim=-1).numpy(), what=f"lse4 b={b} i={i}")


def pin_causal_rule(orc):
    """Query 0 of an s_q = 2 call equals an s_q = 1 call on seqlen - 1 tokens
    with the same query row; query 1 equals an s_q = 1 call on seqlen tokens."""
    inp = mi.small(B=2, s_q=2, H=2, seqlens=[100, 1], seed=17)
    out2, lse2 = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    for i, shift in ((0, 1), (1, 0)):
        q1 = inp.q[:, i:i + 1].clone()
        lens1 = (inp.cache_seqlens - shift).clamp(min=0)
        out1, lse1 = orc.direct(q1, inp.kv_cache, inp.block_table, lens1, inp.scale)
        assert np.array_equal(out1[:, 0], out2[:, i]), f"causal rule, query {i}"
        assert np.array_equal(lse1[:, 0], lse2[:, i]), f"causal rule lse, query {i}"
    assert np.all(out2[1, 0] == 0) and np.all(np.isneginf(lse2[1, 0])), "empty context for query 0"


def pin_paging_invariance(orc):
    """The page table only names where rows live: identity and shuffled tables
    over the same logical rows give bit-identical results."""
    lens = [65, 190, 7]
    ident = mi.small(B=3, s_q=1, H=2, seqlens=lens, table="identity", seed=18)
    shuf = mi.small(B=3, s_q=1, H=2, seqlens=lens, table="shuffled", seed=18)
    # rebuild the shuffled cache so its logical rows equal the identity cache's
    kv = torch.empty_like(ident.kv_cache)
    for b, L in enumerate(lens):
        for p in range((L + 63) // 64):
            kv[int(shuf.block_table[b, p])] = ident.kv_cache[int(ident.block_table[b, p])]
    o1, l1 = orc.direct(ident.q, ident.kv_cache, ident.block_table, ident.cache_seqlens, ident.scale)
    o2, l2 = orc.direct(ident.q, kv, shuf.block_table, shuf.cache_seqlens, ident.scale)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2), "paging changed the result"


def pin_tail_rows_unread(orc):
    """Cache rows past a sequence's length may hold anything (NaN here)."""
    lens = [1, 70, 129]
    clean = mi.small(B=3, s_q=2, H=2, seqlens=lens, seed=19)
    dirty = mi.small(B=3, s_q=2, H=2, seqlens=lens, seed=19, tail_fill=float("nan"))
    assert torch.isnan(dirty.kv_cache.float()).any()
    o1, l1 = orc.direct(clean.q, clean.kv_cache, clean.block_table, clean.cache_seqlens, clean.scale)
    o2, l2 = orc.direct(dirty.q, dirty.kv_cache, dirty.block_table, dirty.cache_seqlens, dirty.scale)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2), "tail rows reached the result"


def pin_transposed_equals_direct(orc):
    """The method's transposed flow gives the direct flow's result (brute
    force on tiny inputs)."""
    for lens, s_q, H in (([1, 3, 8], 1, 4), ([2, 8, 5], 2, 3), ([70, 129], 2, 2)):
        inp = mi.small(B=len(lens), s_q=s_q, H=H, seqlens=lens, seed=20 + len(lens))
        a = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
        t = orc.transposed(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
        _close(t[0], a[0], what="transposed out")
        _close(t[1], a[1], what="transposed lse")


def pin_online_equals_direct(orc):
    """The tiled online-softmax recurrence equals one-shot softmax for any
    tile size."""
    lens = [1, 64, 65, 300]
    inp = mi.small(B=4, s_q=2, H=2, seqlens=lens, seed=24)
    a = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    for tile in (1, 3, 64, 128, 1000):
        o = orc.online(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale, tile)
        _close(o[0], a[0], what=f"online out tile={tile}")
        _close(o[1], a[1], what=f"online lse tile={tile}")


def pin_split_merge_equals_unsplit(orc):
    """Partial results over token ranges merged through their lse equal the
    unsplit result, including empty ranges and ranges past the causal limit."""
    lens = [1, 129, 300]
    inp = mi.small(B=3, s_q=2, H=2, seqlens=lens, seed=25)
    a = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    bounds = np.array([[0, 0, 1, 1, 1],
                       [0, 50, 50, 128, 129],
                       [0, 1, 150, 299, 300]], dtype=np.int64)
    m = orc.split_merge(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale, bounds)
    _close(m[0], a[0], what="split-merge out")
    _close(m[1], a[1], what="split-merge lse")


def pin_outlier_channels(orc):
    """Outlier latent channels (x20 in q and cache) against SDPA: large logits
    and near one-hot softmax stay exact in fp64."""
    inp = mi.small(B=1, s_q=2, H=2, seqlens=[257], outliers=4, seed=26)
    out, lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    q = torch.from_numpy(_bf16_to_f64(inp.q))
    rows = torch.from_numpy(_rows_of(inp, 0, 257))
    for i in range(2):
        n = 256 + i
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[0, i].unsqueeze(1), rows[:n].unsqueeze(0).expand(2, n, 576),
            rows[:n, :512].unsqueeze(0).expand(2, n, 512), scale=inp.scale)
        _close(out[0, i], ref[:, 0].numpy(), rel=1e-11, what="outliers")


def pin_merge_states_closed_forms(orc):
    """Merging partial states: one state is returned as it is; two equal
    states give the same output and lse + ln 2; an empty state (lse = -inf)
    takes no weight; a row whose states are all empty gives 0 and -inf; lse
    is torch's logsumexp of the partial lse values."""
    rng = np.random.default_rng(30)
    parts = rng.standard_normal((3, 5, 512))
    lses = rng.standard_normal((3, 5)) * 4
    out, lse = orc.merge_states(parts[:1], lses[:1])
    assert np.array_equal(out, parts[0]) and np.array_equal(lse, lses[0])
    two = np.stack([parts[0], parts[0]])
    out, lse = orc.merge_states(two, np.stack([lses[0], lses[0]]))
    _close(out, parts[0], what="two equal states")
    _close(lse, lses[0] + math.log(2.0), what="two equal states lse")
    empty = np.array(lses)
    empty[1] = -np.inf
    out, lse = orc.merge_states(parts[:2], empty[:2])
    assert np.array_equal(out, parts[0]) and np.array_equal(lse, lses[0])
    none = np.full((2, 5), -np.inf)
    out, lse = orc.merge_states(parts[:2], none)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    out, lse = orc.merge_states(parts, lses)
    _close(lse, torch.logsumexp(torch.from_numpy(lses), dim=0).numpy(), what="merged lse vs logsumexp")


def pin_merge_states_of_shards_equals_whole(orc):
    """Attention over page-aligned shards of every sequence (each shard a
    problem of its own: the same queries, a slice of the page table), merged
    through the partial lse values, equals attention over the whole
    sequences; shards past a sequence's end are empty."""
    lens = [1, 200, 64 * 7 + 5]
    inp = mi.small(B=3, s_q=1, H=3, seqlens=lens, seed=31)
    whole = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    cuts = [0, 2, 3, 8]  # page boundaries of three shards
    outs, lses = [], []
    for r in range(3):
        p0, p1 = cuts[r], cuts[r + 1]
        sl = torch.tensor([min(max(L - 64 * p0, 0), 64 * (p1 - p0)) for L in lens], dtype=torch.int32)
        bt = inp.block_table[:, p0:p1].contiguous()
        o, l = orc.direct(inp.q, inp.kv_cache, bt, sl, inp.scale)
        outs.append(o)
        lses.append(l)
    out, lse = orc.merge_states(np.stack(outs), np.stack(lses))
    _close(out, whole[0], what="merged shards out")
    _close(lse, whole[1], what="merged shards lse")


def _e4m3_by_torch(codes) -> np.ndarray:
    """Library decoding of e4m3 codes: torch's float8_e4m3fn, widened."""
    c = torch.as_tensor(np.asarray(codes, dtype=np.uint8))
    return c.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def pin_e4m3_decoding(orc):
    """Every e4m3 code decodes as torch's float8_e4m3fn does (NaN codes NaN),
    and spot values of the format: 1.0, 448, 2^-6, 2^-9, -1.0, 0.5, 2.0."""
    codes = np.arange(256, dtype=np.uint8)
    mine = orc.e4m3(codes)
    ref = _e4m3_by_torch(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    assert np.array_equal(mine[~nan], ref[~nan])
    spots = {0x38: 1.0, 0x7E: 448.0, 0x08: 2.0 ** -6, 0x01: 2.0 ** -9, 0xB8: -1.0, 0x30: 0.5, 0x40: 2.0}
    for c, v in spots.items():
        assert orc.e4m3([c])[0] == v, hex(c)


def pin_fp8_cache_equals_exact_bf16_cache(orc):
    """With power-of-two token scales every dequantised value is a bf16 number,
    so attention over the e4m3 cache equals the (pinned) bf16 definition over
    that cache dequantised by torch."""
    inp = mi.small(B=3, s_q=2, H=3, seqlens=[1, 100, 200], seed=33)
    c = mi.fp8_cache(inp.kv_cache.shape[0], seed=34, pow2_scales=True)
    deq = torch.from_numpy(_e4m3_by_torch(c.codes.numpy())) * c.scale.to(torch.float64)[..., None]
    as_bf16 = deq.to(torch.bfloat16)
    assert torch.equal(as_bf16.to(torch.float64), deq)  # exact in bf16
    want = orc.direct(inp.q, as_bf16, inp.block_table, inp.cache_seqlens, inp.scale)
    got = orc.direct_fp8(inp.q, c.codes, c.scale, inp.block_table, inp.cache_seqlens, inp.scale)
    _close(got[0], want[0], what="fp8 out")
    _close(got[1], want[1], what="fp8 lse")


def pin_fp8_cache_against_sdpa(orc):
    """Arbitrary token scales: torch SDPA in float64 on rows dequantised by
    torch (float8_e4m3fn times the token's scale)."""
    inp = mi.small(B=2, s_q=1, H=2, seqlens=[70, 130], seed=35)
    c = mi.fp8_cache(inp.kv_cache.shape[0], seed=36)
    out, lse = orc.direct_fp8(inp.q, c.codes, c.scale, inp.block_table, inp.cache_seqlens, inp.scale)
    deq = torch.from_numpy(_e4m3_by_torch(c.codes.numpy())) * c.scale.to(torch.float64)[..., None]
    q = torch.from_numpy(_bf16_to_f64(inp.q))
    for b, L in enumerate(inp.cache_seqlens.tolist()):
        rows = torch.stack([deq[int(inp.block_table[b, j // 64]), j % 64] for j in range(L)])
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[b, 0].unsqueeze(1), rows.unsqueeze(0).expand(2, L, 576),
            rows[:, :512].unsqueeze(0).expand(2, L, 512), scale=inp.scale)
        _close(out[b, 0], ref[:, 0].numpy(), rel=1e-11, what="fp8 vs sdpa")
        s = (q[b, 0] @ rows.T) * inp.scale
        _close(lse[b, 0], torch.logsumexp(s, dim=-1).numpy(), rel=1e-11, what="fp8 lse vs logsumexp")


def _selection_matrix(H, perm_seed, rng_cols=512):
    """[H, 128, 512] bf16 matrices whose row e of head h has a single 1, in a
    seeded column: decompression then copies 128 chosen latent columns."""
    g = torch.Generator().manual_seed(perm_seed)
    w = torch.zeros(H, 128, rng_cols)
    cols = []
    for h in range(H):
        c = torch.randperm(rng_cols, generator=g)[:128]
        w[h, torch.arange(128), c] = 1.0
        cols.append(c)
    return w.to(torch.bfloat16), cols


def pin_naive_selection_equals_absorbed(orc):
    """Non-absorbed form with up-projections that select latent columns (k_e =
    C[a_e], v_e = C[b_e]) against the absorbed form: absorbing the key matrix
    into the query gives the 576-wide query q~[a_e] = q[e], q~[512 + r] =
    q[128 + r] (exact in bf16), so the scores, hence lse, must agree to
    rounding, and the output must be the absorbed output's columns b_e."""
    lens = [1, 70, 129, 300]
    base = mi.small(B=len(lens), s_q=2, H=3, seqlens=lens, seed=70)
    nv = mi.naive_inputs(len(lens), 2, 3, seed=71)
    w_uk, a_cols = _selection_matrix(3, 72)
    w_uv, b_cols = _selection_matrix(3, 73)
    out, lse = orc.naive(nv.q, base.kv_cache, w_uk, w_uv, base.block_table, base.cache_seqlens, base.scale)
    qt = torch.zeros(len(lens), 2, 3, 576)
    qf = nv.q.to(torch.float32)
    for h in range(3):
        qt[:, :, h, a_cols[h]] = qf[:, :, h, :128]
        qt[:, :, h, 512:] = qf[:, :, h, 128:]
    a_out, a_lse = orc.direct(qt.to(torch.bfloat16), base.kv_cache, base.block_table, base.cache_seqlens,
                              base.scale)
    _close(lse, a_lse, what="naive lse vs absorbed")
    for h in range(3):
        _close(out[:, :, h], a_out[:, :, h][..., b_cols[h].numpy()], what=f"naive out vs absorbed h={h}")


def pin_naive_against_sdpa(orc):
    """Dense random up-projections: keys and values decompressed with torch
    float64 matmuls, then torch's scaled_dot_product_attention and logsumexp;
    ragged lengths, s_q = 2 (query i sees seqlen - 1 + i tokens)."""
    lens = [1, 2, 64, 65, 200]
    base = mi.small(B=len(lens), s_q=2, H=2, seqlens=lens, seed=74)
    nv = mi.naive_inputs(len(lens), 2, 2, seed=75)
    out, lse = orc.naive(nv.q, base.kv_cache, nv.w_uk, nv.w_uv, base.block_table, base.cache_seqlens, base.scale)
    q = torch.from_numpy(_bf16_to_f64(nv.q))
    wk = torch.from_numpy(_bf16_to_f64(nv.w_uk))
    wv = torch.from_numpy(_bf16_to_f64(nv.w_uv))
    for b, L in enumerate(lens):
        rows = torch.from_numpy(_rows_of(base, b, L))
        for i in range(2):
            n = max(0, L - 1 + i)
            if n == 0:
                assert np.all(out[b, i] == 0) and np.all(np.isneginf(lse[b, i])), "empty context"
                continue
            for h in range(2):
                k = torch.cat([rows[:n, :512] @ wk[h].T, rows[:n, 512:]], dim=1)   # [n, 192]
                v = rows[:n, :512] @ wv[h].T                                       # [n, 128]
                qq = q[b, i, h].view(1, 1, 192)
                ref = torch.nn.functional.scaled_dot_product_attention(qq, k.unsqueeze(0), v.unsqueeze(0),
                                                                       scale=base.scale)
                _close(out[b, i, h], ref[0, 0].numpy(), what=f"naive sdpa b={b} i={i} h={h}")
                _close(lse[b, i, h], torch.logsumexp(base.scale * (k @ q[b, i, h]), dim=0).numpy(),
                       what=f"naive lse b={b} i={i} h={h}")


def pin_naive_single_token(orc):
    """A one-token context returns that token's decompressed value exactly
    (numpy matmul of the latent row with the value matrix) and lse = the
    scaled score of its decompressed key."""
    base = mi.small(B=2, s_q=1, H=2, seqlens=[1, 1], seed=76)
    nv = mi.naive_inputs(2, 1, 2, seed=77)
    out, lse = orc.naive(nv.q, base.kv_cache, nv.w_uk, nv.w_uv, base.block_table, base.cache_seqlens, base.scale)
    q = _bf16_to_f64(nv.q)
    wk, wv = _bf16_to_f64(nv.w_uk), _bf16_to_f64(nv.w_uv)
    for b in range(2):
        row = _rows_of(base, b, 1)[0]
        for h in range(2):
            _close(out[b, 0, h], wv[h] @ row[:512], what="single-token value")
            key = np.concatenate([wk[h] @ row[:512], row[512:]])
            _close(lse[b, 0, h], base.scale * float(q[b, 0, h] @ key), what="single-token lse")


ALL_PINS = [
    pin_naive_selection_equals_absorbed, pin_naive_against_sdpa, pin_naive_single_token,
    pin_single_token,
    pin_equal_scores_mean_of_values,
    pin_zero_scale,
    pin_weights_sum_to_one,
    pin_two_token_closed_form,
    pin_torch_sdpa,
    pin_torch_sdpa_four_queries,
    pin_causal_rule,
    pin_paging_invariance,
    pin_tail_rows_unread,
    pin_transposed_equals_direct,
    pin_online_equals_direct,
    pin_split_merge_equals_unsplit,
    pin_outlier_channels,
    pin_merge_states_closed_forms,
    pin_merge_states_of_shards_equals_whole,
    pin_e4m3_decoding,
    pin_fp8_cache_equals_exact_bf16_cache,
    pin_fp8_cache_against_sdpa,
]
