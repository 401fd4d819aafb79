"""Context-parallel decode on the host (no GPU): the page split, and the
gather of partial states over two gloo ranks.

Each rank's attention over its own pages is computed here by the oracle (test
infrastructure) in place of the GPU kernel; the product code under test is the
split (``local_shard``) and the exchange (``gather_states``).  The merged
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


def test_local_shards_partition_the_tokens():
    import mla_inputs as mi
    from decode_attention_latent_b200.context_parallel import local_shard
    inp = mi.small(B=4, s_q=1, H=2, seqlens=[1, 64, 65, 64 * 9 + 3], seed=40)
    for W in (1, 2, 3, 5):
        seen = {}
        for r in range(W):
            sl, bt = local_shard(inp.cache_seqlens, inp.block_table, W, r)
            for b in range(4):
                for j in range(int(sl[b])):
                    seen.setdefault((b, int(bt[b, j // 64]), j % 64), []).append(r)
        want = {(b, int(inp.block_table[b, j // 64]), j % 64) for b, L in enumerate(inp.cache_seqlens.tolist())
                for j in range(L)}
        assert set(seen) == want and all(len(v) == 1 for v in seen.values())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path[:0] = [ROOT, HERE]
    import torch.distributed as dist
    import mla_inputs as mi
    import oracle
    from decode_attention_latent_b200.context_parallel import gather_states, local_shard
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = mi.small(B=3, s_q=1, H=4, seqlens=[70, 1, 64 * 5 + 9], seed=41)
        orc = oracle.default()
        sl, bt = local_shard(inp.cache_seqlens, inp.block_table, world, rank)
        o, l = orc.direct(inp.q, inp.kv_cache, bt, sl, inp.scale)
        # what the GPU decode would hand over: bf16 out, fp32 lse
        out = torch.from_numpy(o).to(torch.bfloat16)
        lse = torch.from_numpy(l).to(torch.float32)
        out_parts, lse_parts = gather_states(out, lse)
        assert out_parts.shape == (world,) + tuple(out.shape) and out_parts.dtype == torch.bfloat16
        assert torch.equal(out_parts[rank], out) and torch.equal(lse_parts[rank], lse)
        m_out, m_lse = orc.merge_states(out_parts, lse_parts)
        w_out, w_lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(w_out), 1e-30))) - 7)
        result[rank] = (float(np.max(np.abs(m_out - w_out) / (1.5e-2 + ulp))),
                        float(np.max(np.abs(m_lse - w_lse))))
    finally:
        dist.destroy_process_group()


def test_gather_and_merge_over_two_gloo_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    result = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, result)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    for r in range(2):
        err_out, err_lse = result[r]
        assert err_out <= 1.0 and err_lse <= 1e-3, result[r]
