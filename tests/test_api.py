"""The C-ABI library on the host (no GPU): it loads, exports every symbol the
header declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

import decode_attention_latent_b200 as mla
from decode_attention_latent_b200 import build as mla_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla_decode.h")


@pytest.fixture(scope="module")
def lib():
    mla_build.build()
    return mla.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("mla_decode", "mla_decode_metadata", "mla_decode_combine", "mla_decode_workspace_size",
              "mla_sched_meta_ints", "mla_get_device_error", "mla_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} missing from {mla.library_path()}"
    assert set(declared_functions()) <= set(mla.EXPORTED)


def test_status_strings(lib):
    for code, name in mla.STATUS_NAMES.items():
        assert lib.mla_status_string(code).decode() == name


def test_sizes(lib):
    assert lib.mla_sched_meta_ints(148) == 16 + 8 * 148
    assert lib.mla_sched_meta_ints(0) == 0
    # pieces = (B + tuples) * G; each holds s_q * HG rows of 512 fp32 + lse
    ws = lib.mla_decode_workspace_size(8, 1, 16, 148)
    pieces = 8 + 148
    assert ws >= pieces * 16 * 512 * 4 + pieces * 16 * 4
    ws128 = lib.mla_decode_workspace_size(64, 1, 128, 148)
    assert ws128 >= (64 + 74) * 2 * 64 * 513 * 4
    for bad in ((8, 3, 16, 148), (8, 1, 24, 148), (0, 1, 16, 148), (8, 1, 128, 1), (5000, 1, 16, 148)):
        assert lib.mla_decode_workspace_size(*bad) == 0, bad


P = ctypes.c_void_p
GOOD = 0x100000  # aligned fake addresses: validation never dereferences them


def decode_args(**kw):
    a = dict(q=GOOD, kv=GOOD, bt=GOOD, sl=GOOD, B=8, s_q=1, H=16, nb=1024, mb=1024, scale=0.07,
             sms=148, sched=GOOD, splits=GOOD, ws=GOOD, wsb=1 << 30, out=GOOD, lse=GOOD)
    a.update(kw)
    return [P(a["q"]), P(a["kv"]), P(a["bt"]), P(a["sl"]), a["B"], a["s_q"], a["H"], a["nb"], a["mb"],
            ctypes.c_float(a["scale"]), a["sms"], P(a["sched"]), P(a["splits"]), P(a["ws"]), a["wsb"],
            P(a["out"]), P(a["lse"]), P(0)]


@pytest.mark.parametrize("kw,status", [
    (dict(q=0), 1), (dict(kv=0), 1), (dict(out=0), 1), (dict(ws=0), 1),
    (dict(B=0), 1), (dict(nb=0), 1), (dict(mb=0), 1), (dict(scale=float("nan")), 1),
    (dict(s_q=3), 3), (dict(H=24), 3), (dict(H=128, sms=1), 3),
    (dict(q=GOOD + 2), 2), (dict(kv=GOOD + 8), 2), (dict(ws=GOOD + 16), 2), (dict(lse=GOOD + 2), 2),
    (dict(wsb=1024), 4),
])
def test_decode_rejects_bad_arguments(lib, kw, status):
    assert lib.mla_decode(*decode_args(**kw)) == status


def test_metadata_rejects_bad_arguments(lib):
    assert lib.mla_decode_metadata(P(0), 8, 1, 16, 148, P(GOOD), P(GOOD), P(0)) == 1
    assert lib.mla_decode_metadata(P(GOOD), 0, 1, 16, 148, P(GOOD), P(GOOD), P(0)) == 1
    assert lib.mla_decode_metadata(P(GOOD), 8, 2, 48, 148, P(GOOD), P(GOOD), P(0)) == 3
    assert lib.mla_decode_metadata(P(GOOD + 1), 8, 1, 16, 148, P(GOOD), P(GOOD), P(0)) == 2


def test_combine_rejects_bad_arguments(lib):
    args = [P(GOOD), P(GOOD), P(GOOD), 1 << 30, 8, 1, 16, 148, P(GOOD), P(GOOD), P(0)]
    bad = list(args); bad[0] = P(0)
    assert lib.mla_decode_combine(*bad) == 1
    bad = list(args); bad[3] = 16
    assert lib.mla_decode_combine(*bad) == 4
    bad = list(args); bad[5] = 3  # s_q = 3 is outside the supported set
    assert lib.mla_decode_combine(*bad) == 3


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(mla.MLAError):
        mla.load_library(str(tmp_path / "missing.so"))


def test_merge_states_rejects_bad_arguments(lib):
    args = [P(GOOD), P(GOOD), 4, 128, P(GOOD), P(GOOD), P(0)]
    for i, v, status in ((0, P(0), 1), (1, P(0), 1), (4, P(0), 1), (5, P(0), 1), (2, 0, 1), (2, 65, 1),
                         (3, 0, 1), (3, 1 << 31, 1), (0, P(GOOD + 8), 2), (4, P(GOOD + 8), 2),
                         (1, P(GOOD + 2), 2), (5, P(GOOD + 1), 2)):
        bad = list(args)
        bad[i] = v
        assert lib.mla_merge_states(*bad) == status, (i, v)


def test_decode_fp8_rejects_bad_arguments(lib):
    def args(**kw):
        a = dict(q=GOOD, codes=GOOD, scale=GOOD, bt=GOOD, sl=GOOD, B=8, s_q=1, H=16, nb=1024, mb=1024, sms=148)
        a.update(kw)
        return [P(a["q"]), P(a["codes"]), P(a["scale"]), P(a["bt"]), P(a["sl"]), a["B"], a["s_q"], a["H"],
                a["nb"], a["mb"], ctypes.c_float(0.07), a["sms"], P(GOOD), P(GOOD), P(GOOD), 1 << 30,
                P(GOOD), P(GOOD), P(0)]
    assert lib.mla_decode_fp8(*args(codes=0)) == 1
    assert lib.mla_decode_fp8(*args(scale=0)) == 1
    assert lib.mla_decode_fp8(*args(H=64)) == 3      # 16 or 32 query columns only
    assert lib.mla_decode_fp8(*args(H=16, s_q=4)) == 3
    assert lib.mla_decode_fp8(*args(s_q=2, H=8)) == 3
    assert lib.mla_decode_fp8(*args(codes=GOOD + 8)) == 2
    assert lib.mla_decode_fp8(*args(scale=GOOD + 4)) == 2
