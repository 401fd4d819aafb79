"""Failure detection on the GPU without a fault.

A CTA whose first cache load is announced but never issued (the library's
mla_debug_stall_cta test hook) must end its bounded waits after their time
limit, report MLA_DEVERR_TIMEOUT in the device error word, release its TMEM
and exit; the context must stay usable, so the next call on the same process
(after mla_decode_metadata has reset sched_meta, as the header asks after a
device error) returns a clean error word and results equal to the oracle's.
Both the bf16 kernel and the FP8-cache kernel (whose first staging unit is the
one withheld) are checked.  Each check runs in a child process so the hook
never reaches other tests.  Invalid data (a bad page-table entry, a schedule
built for another shape, a stale completion counter) is covered in
test_parity.py.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import os, sys
sys.path.insert(0, ROOT)
import numpy as np
import torch
import decode_attention_latent_b200 as mla
import mla_inputs as mi
import oracle

dev = torch.device("cuda", 0)
inp = mi.small(B=3, s_q=1, H=16, seqlens=[900, 300, 2000], seed=900)
q, kv, bt, sl = (x.to(dev) for x in (inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens))
if FP8:
    cache = mi.fp8_cache(inp.kv_cache.shape[0], seed=901)
    codes, scales = cache.codes.to(dev), cache.scale.to(dev)


def run():
    sched, splits = mla.decode_metadata(sl, 1, 16, 8)
    if FP8:
        out, lse = mla.decode_fp8(q, codes, scales, bt, sl, inp.scale, sched_meta=sched, num_splits=splits,
                                  num_sms_=8)
    else:
        out, lse = mla.decode(q, kv, bt, sl, inp.scale, sched_meta=sched, num_splits=splits, num_sms_=8)
    return out, lse, mla.get_device_error(sched)


mla.debug_stall_cta(3)   # CTA 3 of 8 owns tiles 12..15 of the 27
_, _, err = run()
print("stalled call error word", err)
assert err & mla.DEVERR_TIMEOUT, err
mla.debug_stall_cta(-1)
out, lse, err = run()
assert err == 0, err
orc = oracle.default()
if FP8:
    ref_out, ref_lse = orc.direct_fp8(inp.q, cache.codes, cache.scale, inp.block_table, inp.cache_seqlens,
                                      inp.scale)
else:
    ref_out, ref_lse = orc.direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale)
g_out = out.float().cpu().numpy()
g_lse = lse.cpu().numpy()
ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref_out), 1e-30))) - 7)  # one bf16 ulp
assert np.all(np.abs(g_out - ref_out) <= 1.5e-2 + ulp), np.abs(g_out - ref_out).max()
assert np.abs(g_lse - ref_lse).max() <= 1e-3
print("ok")
'''


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "fp8"])
def test_stalled_cta_times_out_and_context_survives(fp8):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\nFP8 = {fp8!r}\n" + CHILD], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
