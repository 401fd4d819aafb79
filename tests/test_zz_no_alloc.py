"""The no-allocation entry point, mla_decode_static_workspace, against
mla_decode (GPU, through the C ABI).

Some callers cannot hand the library a scratch buffer: code whose device
memory is reserved up front by its own pool, or a plugin inside a framework
that owns every device allocation.  For them the library carries a fixed
device workspace (MLA_STATIC_WORKSPACE_BYTES) and this entry point uses it
instead of a caller-supplied one.  The test checks that two calls in a row
give the results of the ordinary entry point (same tolerance as the parity
tests), and that a shape too large for the built-in workspace is refused
before anything is launched.  It lives in its own file so that pytest
collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_attention_latent_b200 as mla
import mla_inputs as mi

pytestmark = pytest.mark.gpu

ATOL = 1.5e-2
LSE_ATOL = 1e-3
STATIC_BYTES = 8 << 20  # MLA_STATIC_WORKSPACE_BYTES
P = ctypes.c_void_p


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


def _call_static(lib, t, n_sms, sched, splits, out, lse):
    return lib.mla_decode_static_workspace(
        P(t["q"].data_ptr()), P(t["kv"].data_ptr()), P(t["bt"].data_ptr()), P(t["sl"].data_ptr()),
        t["B"], t["s_q"], t["H"], t["kv"].shape[0], t["bt"].shape[1], ctypes.c_float(t["scale"]), n_sms,
        P(sched.data_ptr()), P(splits.data_ptr()), P(out.data_ptr()), P(lse.data_ptr()),
        P(torch.cuda.current_stream().cuda_stream))


def _close(a_out, a_lse, b_out, b_lse):
    a_out, b_out = a_out.float().cpu().numpy(), b_out.float().cpu().numpy()
    a_lse, b_lse = a_lse.cpu().numpy(), b_lse.cpu().numpy()
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(b_out), 1e-30))) - 7)  # one bf16 ulp
    bound = np.where(np.abs(b_out) < 1.0, ATOL, ATOL + ulp)  # the parity tests' bound
    assert np.all(np.abs(a_out - b_out) <= bound)
    fin = np.isfinite(b_lse)
    assert np.array_equal(np.isfinite(a_lse), fin)
    assert np.all(np.abs(a_lse[fin] - b_lse[fin]) <= LSE_ATOL)


# (s_q, H, lengths, CTAs): the workspace grows with the pieces a call can
# produce, (B + CTAs) x the query columns of a CTA, so the wider shapes run on
# fewer CTAs to stay inside the built-in 8 MiB.
CASES = {
    # B=8, s_q=1, H=16 with empty, one-token and ragged sequences (about 5.1 MB at 148 CTAs)
    "b8_sq1_h16": (1, 16, [8192, 5000, 129, 1, 0, 3000, 64, 7000], None),
    # two query positions (causal rule, 32 query columns per CTA): about 4.4 MB at 64 CTAs
    "b4_sq2_h16": (2, 16, [4000, 1, 700, 2600], 64),
    # 64 heads in one group of 64 query columns: about 6.4 MB at 48 CTAs
    "b2_sq1_h64": (1, 64, [3000, 900], 48),
    # the largest batch of 16-head sequences whose workspace fits at 148 CTAs
    "largest_fit": (1, 16, None, None),
}


def _largest_batch_that_fits(lib, n_sms):
    B = 1
    while B < 4096 and lib.mla_decode_workspace_size(B + 1, 1, 16, n_sms) <= STATIC_BYTES:
        B += 1
    return B


@pytest.mark.parametrize("case", list(CASES))
def test_static_workspace_matches_mla_decode_twice(dev, case):
    lib = mla.load_library()
    s_q, H, lens, n_sms = CASES[case]
    n_sms = mla.num_sms(dev) if n_sms is None else n_sms
    if lens is None:
        B = _largest_batch_that_fits(lib, n_sms)
        lens = [int(x) for x in np.random.default_rng(7).integers(0, 3000, B)]
    inp = mi.small(B=len(lens), s_q=s_q, H=H, seqlens=lens, seed=900, tail_fill=float("nan"))
    t = dict(q=inp.q.to(dev), kv=inp.kv_cache.to(dev), bt=inp.block_table.to(dev),
             sl=inp.cache_seqlens.to(dev), B=inp.B, s_q=inp.s_q, H=inp.H, scale=inp.scale)
    assert lib.mla_decode_workspace_size(t["B"], t["s_q"], t["H"], n_sms) <= STATIC_BYTES
    sched, splits = mla.decode_metadata(t["sl"], t["s_q"], t["H"], n_sms)
    ref_out, ref_lse = mla.decode(t["q"], t["kv"], t["bt"], t["sl"], t["scale"], sched_meta=sched,
                                  num_splits=splits, num_sms_=n_sms)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full((t["B"], t["s_q"], t["H"], 512), float("nan"), dtype=torch.bfloat16, device=dev)
        lse = torch.full((t["B"], t["s_q"], t["H"]), float("nan"), dtype=torch.float32, device=dev)
        rc = _call_static(lib, t, n_sms, sched, splits, out, lse)
        assert rc == 0, lib.mla_last_error_message().decode()
        torch.cuda.synchronize()
        assert mla.get_device_error(sched) == 0
        _close(out, lse, ref_out, ref_lse)


def test_static_workspace_refuses_oversized_shapes(dev):
    lib = mla.load_library()
    n_sms = mla.num_sms(dev)
    B, s_q, H = 64, 1, 128
    assert lib.mla_decode_workspace_size(B, s_q, H, n_sms) > STATIC_BYTES
    g = 1 << 20  # aligned stand-in addresses: the size check returns before any use
    rc = lib.mla_decode_static_workspace(P(g), P(g), P(g), P(g), B, s_q, H, 1024, 1024, ctypes.c_float(0.07),
                                         n_sms, P(g), P(g), P(g), P(g), P(0))
    assert rc == 4  # MLA_ERR_WORKSPACE_TOO_SMALL
    assert b"static" in lib.mla_last_error_message() or b"built-in" in lib.mla_last_error_message()
