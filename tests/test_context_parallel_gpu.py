"""Context-parallel decode on the GPU: the merge kernel against the oracle's
merge, and W ranks emulated one after another on one device (each runs the
decode on its own pages; no rank waits on another) merged and compared with
the oracle over the whole sequences."""
import os
import socket

import numpy as np
import pytest
import torch

import decode_attention_latent_b200 as mla
import mla_inputs as mi
import oracle
from decode_attention_latent_b200.context_parallel import decode_context_parallel, decode_local_state, local_shard
from test_parity import compare, ulp_bf16

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


@pytest.mark.parametrize("W,rows", [(1, 7), (2, 33), (5, 129), (64, 3)])
def test_merge_states_matches_oracle(dev, orc, W, rows):
    g = torch.Generator().manual_seed(50 + W)
    parts = torch.randn(W, rows, 512, generator=g).to(torch.bfloat16)
    lses = (torch.randn(W, rows, generator=g) * 6).to(torch.float32)
    lses[0, 0] = -float("inf")            # one empty state
    if W > 1:
        lses[:, 1] = -float("inf")        # a row with no state at all
    out, lse = mla.merge_states(parts.to(dev), lses.to(dev))
    r_out, r_lse = orc.merge_states(parts, lses)
    g_out = out.float().cpu().numpy()
    g_lse = lse.cpu().numpy()
    fin = np.isfinite(r_lse)
    assert np.array_equal(np.isfinite(g_lse), fin)
    assert np.all(g_out[~fin] == 0)
    assert np.all(np.abs(g_out - r_out) <= ulp_bf16(r_out) + 1e-6)
    assert np.abs(g_lse[fin] - r_lse[fin]).max() <= 1e-5


@pytest.mark.parametrize("H,W,s_q", [(16, 2, 1), (16, 3, 1), (16, 8, 1), (128, 2, 1),
                                     (16, 2, 2), (16, 3, 4), (32, 3, 2), (16, 8, 8), (64, 2, 2)])
def test_emulated_ranks_match_oracle(dev, orc, H, W, s_q):
    # lengths below s_q - 1, at page edges and long; every rank's state from
    # decode_local_state (the causal query on the last rank, folded before it)
    inp = mi.small(B=5, s_q=s_q, H=H, seqlens=[1, 66, 129, 700, 64 * 20 + 5], seed=51)
    q, kv = inp.q.to(dev), inp.kv_cache.to(dev)
    outs, lses = [], []
    for r in range(W):
        sl, bt = local_shard(inp.cache_seqlens, inp.block_table, W, r, s_q)
        o, l = decode_local_state(q, kv, bt.to(dev), sl.to(dev), inp.scale, r == W - 1)
        outs.append(o)
        lses.append(l)
    out, lse = mla.merge_states(torch.stack(outs), torch.stack(lses))
    r_out, r_lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
    compare(out.float().cpu().numpy(), lse.cpu().numpy(), r_out, r_lse,
            what=f"context-parallel W={W} s_q={s_q} H={H}")


def test_one_rank_nccl_group_is_plain_decode(dev):
    # gather over NCCL and merge of a single state: the plain decode, bit for bit
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    inp = mi.small(B=2, s_q=1, H=16, seqlens=[300, 1000], seed=52)
    q, kv, bt, sl = (x.to(dev) for x in (inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens))
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=dev)
    try:
        out, lse = decode_context_parallel(q, kv, bt, sl, inp.scale)
    finally:
        dist.destroy_process_group()
    ref_out, ref_lse = mla.decode(q, kv, bt, sl, inp.scale)
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


def test_too_many_query_columns_are_refused(dev):
    # s_q > 1 folds the positions into heads before the last rank: s_q H <= 128
    inp = mi.small(B=1, s_q=2, H=128, seqlens=[100], seed=53)
    with pytest.raises(ValueError):
        decode_context_parallel(inp.q.to(dev), inp.kv_cache.to(dev), inp.block_table.to(dev),
                                inp.cache_seqlens.to(dev), inp.scale)
