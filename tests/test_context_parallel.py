"""Context-parallel decode on the host (no GPU): the page split, and the
gather of partial states over two gloo ranks.

Each rank's attention over its own pages is computed here by the oracle (test
infrastructure) in place of the GPU kernel; the product code under test is the
split (``local_shard``), the query each rank decodes (``query_view``) and the
exchange (``gather_states``).  The merged
result must equal the oracle over the whole sequences."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))


def test_page_cuts_cover_every_page_once():
    from decode_attention_latent_b200.context_parallel import page_cuts
    for pages in (0, 1, 2, 7, 64, 1025):
        for W in (1, 2, 3, 8):
            cuts = [page_cuts(pages, W, r) for r in range(W)]
            assert cuts[0][0] == 0 and cuts[-1][1] == pages
            for (a0, a1), (b0, b1) in zip(cuts, cuts[1:]):
                assert a1 == b0 and a0 <= a1
            sizes = [p1 - p0 for p0, p1 in cuts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        page_cuts(4, 2, 2)


@pytest.mark.parametrize("s_q", [1, 2, 8])
def test_local_shards_partition_the_tokens(s_q):
    # every token on exactly one rank; with s_q > 1, every token some query
    # position does not see (the last s_q - 1) on the last rank
    import mla_inputs as mi
    from decode_attention_latent_b200.context_parallel import local_shard
    lens = [1, 3, 64, 65, 66, 128, 129, 64 * 9 + 3]
    inp = mi.small(B=len(lens), s_q=1, H=2, seqlens=lens, seed=40)
    for W in (1, 2, 3, 5):
        seen = {}
        for r in range(W):
            sl, bt = local_shard(inp.cache_seqlens, inp.block_table, W, r, s_q)
            for b in range(len(lens)):
                for j in range(int(sl[b])):
                    seen.setdefault((b, int(bt[b, j // 64]), j % 64), []).append(r)
        want = {(b, int(inp.block_table[b, j // 64]), j % 64) for b, L in enumerate(lens) for j in range(L)}
        assert set(seen) == want and all(len(v) == 1 for v in seen.values())
        for (b, blk, off), ranks in seen.items():
            j = inp.block_table[b].tolist().index(blk) * 64 + off  # global token index
            if j >= lens[b] - s_q + 1:
                assert ranks == [W - 1], (W, b, j)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result, s_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path[:0] = [ROOT, HERE]
    import torch.distributed as dist
    import mla_inputs as mi
    import oracle
    from decode_attention_latent_b200.context_parallel import gather_states, local_shard, query_view
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = mi.small(B=3, s_q=s_q, H=4, seqlens=[70, 1, 64 * 5 + 9], seed=41)
        orc = oracle.default()
        sl, bt = local_shard(inp.cache_seqlens, inp.block_table, world, rank, s_q)
        # this rank's query as the product decodes it (folded into heads before the last rank)
        qv, back = query_view(inp.q, rank == world - 1)
        o, l = orc.direct(qv, inp.kv_cache, bt, sl, inp.scale)
        # what the GPU decode would hand over: bf16 out, fp32 lse
        out, lse = back(torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(l).to(torch.float32))
        out_parts, lse_parts = gather_states(out, lse)
        assert out_parts.shape == (world,) + tuple(out.shape) and out_parts.dtype == torch.bfloat16
        assert torch.equal(out_parts[rank], out) and torch.equal(lse_parts[rank], lse)
        m_out, m_lse = orc.merge_states(out_parts, lse_parts)
        w_out, w_lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(w_out), 1e-30))) - 7)
        fin = np.isfinite(w_lse)  # a query position that sees no token has lse -inf
        assert np.array_equal(np.isfinite(m_lse), fin)
        result[rank] = (float(np.max(np.abs(m_out - w_out) / (1.5e-2 + ulp))),
                        float(np.max(np.abs(m_lse[fin] - w_lse[fin]))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("s_q", [1, 2])
def test_gather_and_merge_over_two_gloo_ranks(s_q):
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    result = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, result, s_q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    for r in range(2):
        err_out, err_lse = result[r]
        assert err_out <= 1.0 and err_lse <= 1e-3, result[r]
