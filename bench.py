"""Benchmark of absorbed-form MLA decode on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one decode call of the workload through the C ABI: the split-KV
metadata kernel, the attention kernel and the combine kernel, on inputs that
are already resident in HBM.  The default workload is the 64K-context,
16-head configuration (B = 8, s_q = 1, H = 16, L = 65536, 604 MB of cache).
The inputs are larger than the 126 MB L2 and consecutive steps read two
different device copies of the cache, so no step can find the cache in L2.

Printed (rank 0, one JSON line): metric / value / unit (microseconds per call,
lower is better), the kernel's roofline against the measured HBM copy
bandwidth, the error against the fp64 oracle on sampled sequences, an
end-to-end figure through the same C ABI with the step's inputs copied from
pinned host memory and its outputs copied back inside the timed region, the
SM clocks sampled during the timed region, and the fp64 CPU oracle timed on a
bounded sample as a baseline.

With N > 1 (launched by torchrun) every rank runs its own replica of the
workload on its own GPU (independent batches, no collective on the data
path); the step time is the max over ranks.  ``--impl reference`` times the
CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import mla_inputs as mi  # noqa: E402

METRIC = "MLA decode µs/call, achieved HBM TB/s and % roofline at 64K ctx, 16 heads"
UNIT = "us/call"
KERNEL_SOURCES = [os.path.join(ROOT, "decode_attention_latent_b200", "csrc", "mla_decode.cu"),
                  os.path.join(ROOT, "decode_attention_latent_b200", "csrc", "sm100_ptx.cuh")]
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 << 20


def kv_copy_count(kv_bytes: int, l2_bytes: int) -> int:
    """Device copies of the cache that consecutive steps cycle through: at
    least two, and enough that a step's cache was last read at least three
    L2 capacities of traffic earlier (so it cannot be found in L2)."""
    return max(2, -(-3 * l2_bytes // max(1, kv_bytes)))


# ---------------------------------------------------------------- helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend=backend, timeout=timedelta(seconds=120))


def max_over_ranks(x: float, device) -> float:
    """Maximum of a per-rank scalar (identity without a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        if device.type == "cuda":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def measured_peaks():
    """(HBM GB/s, its source, bf16 TFLOP/s burst, its source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return (float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy)",
                float(d["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst)")
    except Exception:
        return (FALLBACK_HBM_GBS, "fallback (6.65 TB/s earlier pool measurement)",
                FALLBACK_BF16_TFLOPS, "fallback (1.59 PFLOP/s earlier pool measurement)")


def attention_kernel_name(s_q: int, H: int) -> str:
    """The attention kernel instance the library launches for this shape:
    N = s_q * H query columns per CTA, at most 64."""
    return f"mla_decode_kernel<{min(s_q * H, 64)},{s_q},false>"


def sustained_tflops() -> float:
    """bf16 GEMM throughput sustained under the power cap (MEASURED_PEAKS.json),
    else the earlier pool measurement."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        return 1400.0


def roofline(alg_bytes: int, alg_flops: int, seconds: float, peaks) -> dict:
    """Roofline of one attention launch: the bound is whichever of the HBM
    time (algorithmic bytes / copy bandwidth) and the tensor time
    (algorithmic FLOPs / bf16 GEMM peak) is longer."""
    hbm, hbm_src, tc, tc_src = peaks
    t_hbm = alg_bytes / (hbm * 1e9)
    t_tc = alg_flops / (tc * 1e12)
    both = {"hbm_frac": t_hbm / seconds, "tensor_frac": t_tc / seconds,
            "t_hbm_us": t_hbm * 1e6, "t_tensor_us": t_tc * 1e6}
    if t_tc > t_hbm:
        a = alg_flops / seconds / 1e12
        return {"bound": "tensor", "achieved": a, "peak": tc, "unit": "TFLOP/s", "frac": a / tc,
                "peak_source": tc_src, "both": both}
    a = alg_bytes / seconds / 1e9
    return {"bound": "hbm", "achieved": a, "peak": hbm, "unit": "GB/s", "frac": a / hbm,
            "peak_source": hbm_src, "both": both}


def source_digest() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu summary, if it
    was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"mla_decode_attention_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_b = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_s = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    if not m_b or not m_s or m_s.group(1) != source_digest():
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.count(",") >= 9]
        os.unlink(self.file.name)
        samples = []
        for r in rows:
            try:
                ts = time.mktime(time.strptime(r[0].strip().split(".")[0], "%Y/%m/%d %H:%M:%S"))
                samples.append((ts, [x.strip() for x in r]))
            except Exception:
                continue
        inside = [s for ts, s in samples if t0 - 1.0 <= ts <= t1 + 1.0] or [s for _, s in samples]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(s[2]) for s in inside]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for s in inside:
            for k, name in enumerate(names):
                if s[6 + k].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(inside[0][3]),
                "reasons": sorted(reasons), "samples": len(inside),
                "power_w_max": max(float(s[4]) for s in inside)}


# ------------------------------------------------------------- CPU oracle
def oracle_sample_seconds(orc, inp: mi.Inputs, seqs, tokens: int):
    """Time the oracle on sequences `seqs`, each truncated to `tokens` tokens."""
    sub_len = inp.cache_seqlens.clone()
    sub_len[:] = torch.clamp(sub_len, max=tokens)
    t0 = time.perf_counter()
    orc.direct(inp.q, inp.kv_cache, inp.block_table, sub_len, inp.scale, seqs=list(seqs))
    return time.perf_counter() - t0


def cpu_baseline(inp: mi.Inputs, target_s: float = 15.0):
    """fp64 oracle on a bounded sample of the workload, scaled to one call.
    The oracle's cost is proportional to (output rows) x (tokens)."""
    import oracle
    orc = oracle.default()
    full_tokens = int(inp.cache_seqlens.max())
    tokens = min(full_tokens, 4096)
    t = oracle_sample_seconds(orc, inp, [0], tokens)
    # grow the sample toward the target: first tokens, then sequences
    if t > 0 and tokens < full_tokens:
        tokens = min(full_tokens, max(tokens, int(tokens * (target_s / 2) / t)))
        t = oracle_sample_seconds(orc, inp, [0], tokens)
    n_seq = 1
    if t > 0 and tokens == full_tokens:
        n_seq = max(1, min(inp.B, int(target_s / t)))
        if n_seq > 1:
            t = oracle_sample_seconds(orc, inp, list(range(n_seq)), tokens)
    work_full = sum(int(x) for x in inp.cache_seqlens)
    work_sample = n_seq * tokens
    per_call_s = t * work_full / work_sample
    return {"value": per_call_s * 1e6, "unit": UNIT, "cores": orc.threads(), "kind": "oracle",
            "sample": f"{n_seq} of {inp.B} sequences x {tokens} of {full_tokens} tokens, all "
                      f"{inp.s_q * inp.H} query rows each, {t:.2f} s, scaled by {work_full / work_sample:.1f}"}


def selected_workload(args) -> mi.Workload:
    """The workload named on the command line, with its batch cut to
    ``--batch`` sequences when given (a smaller case of the same shape and
    length distribution, for profiler captures that must stay small)."""
    w = mi.WORKLOADS[args.workload]
    if args.batch:
        if not 1 <= args.batch <= w.B:
            raise SystemExit(f"--batch must be in [1, {w.B}] for {w.name}")
        w = mi.workload(args.workload, B=args.batch)
    return w


def run_reference(args, world, rank):
    """The CPU oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return 0
    import oracle
    w = selected_workload(args)
    inp = mi.make_inputs(w, seed=0)
    orc = oracle.default()
    full_tokens = int(inp.cache_seqlens.max())
    # each step: sequence 0 truncated so the whole run stays within ~2 minutes
    per_step = 120.0 / max(1, args.steps + args.warmup)
    tokens = 256
    t = oracle_sample_seconds(orc, inp, [0], tokens)
    if t > 0:
        tokens = int(max(64, min(full_tokens, tokens * per_step / t)))
    for _ in range(args.warmup):
        oracle_sample_seconds(orc, inp, [0], tokens)
    times = [oracle_sample_seconds(orc, inp, [0], tokens) for _ in range(args.steps)]
    scale = sum(int(x) for x in inp.cache_seqlens) / tokens
    value = statistics.mean(times) * scale * 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(times) * 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": args.workload, "B": w.B, "s_q": w.s_q, "H": w.H,
                                        "seqlen": w.seqlen, "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": orc.threads(), "kind": "oracle",
                         "sample": f"sequence 0 of {w.B}, first {tokens} of {full_tokens} tokens, "
                                   f"{w.s_q * w.H} query rows; scaled by {scale:.1f} per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- GPU arm
# sequences the oracle recomputes for the accuracy figures of each workload
ACCURACY_SAMPLE = {
    "b1_h16_l1k_identity": None,
    "b16_h16_l4k": None,
    "b32_sq2_h16_l16k_outliers": [0, 13, 31],
    "b64_h128_lvar1k32k": [0, 7, 33, 63],
    "b8_h16_l64k": [0, 5],
}


def accuracy(g_out, g_lse, r_out, r_lse, seqs, B):
    """Error of the GPU result against the fp64 oracle on sampled sequences:
    max |out err|, relative RMSE sqrt(sum err^2 / sum ref^2) over those
    outputs, and max |lse err| (the figures and bounds the tests assert)."""
    import numpy as np
    if seqs is not None:
        g_out, g_lse, r_out, r_lse = g_out[seqs], g_lse[seqs], r_out[seqs], r_lse[seqs]
    err = np.abs(g_out.astype(np.float64) - r_out)
    den = float(np.sum(r_out ** 2))
    fin = np.isfinite(r_lse)
    lerr = float(np.abs(g_lse[fin] - r_lse[fin]).max()) if fin.any() else 0.0
    rmse = (float(np.sum(err ** 2)) / den) ** 0.5 if den > 0 else 0.0
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(r_out), 1e-30))) - 7)
    bound = np.where(np.abs(r_out) < 1.0, 1.5e-2, 1.5e-2 + ulp)
    return {"sequences": "all" if seqs is None else f"{len(seqs)} of {B}: {seqs}",
            "out_max_abs_err": float(err.max()), "out_rel_rmse": rmse, "lse_max_abs_err": lerr,
            "out_max_abs_ref": float(np.abs(r_out).max()),
            "within_bounds": bool(np.all(err <= bound) and rmse <= 5e-3 and lerr <= 1e-3),
            "bounds": "out: 1.5e-2 where |ref| < 1, else 1.5e-2 + one bf16 ulp; rel RMSE 5e-3; lse 1e-3"}


def run_ours(args, world, rank, local):
    import ctypes

    import decode_attention_latent_b200 as mla

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl")
    lib = mla.load_library()
    w = selected_workload(args)
    inp = mi.make_inputs(w, seed=rank)
    B, s_q, H = w.B, w.s_q, w.H
    n_sms = mla.num_sms(dev)

    q = inp.q.to(dev)
    kv_bytes = int(inp.kv_cache.numel() * 2)
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", L2_BYTES) or L2_BYTES)
    n_copies = kv_copy_count(kv_bytes, l2)
    kv_copies = [inp.kv_cache.to(dev) for _ in range(n_copies)]
    kv = kv_copies[0]
    bt = inp.block_table.to(dev)
    sl = inp.cache_seqlens.to(dev)
    sched = torch.empty(mla.sched_meta_ints(n_sms), dtype=torch.int32, device=dev)
    splits = torch.empty(B + 1, dtype=torch.int32, device=dev)
    ws_bytes = mla.workspace_size(B, s_q, H, n_sms)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.empty(B, s_q, H, mi.D_V, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, s_q, H, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    P = ctypes.c_void_p

    def call_metadata(st=None):
        rc = lib.mla_decode_metadata(P(sl.data_ptr()), B, s_q, H, n_sms, P(sched.data_ptr()),
                                     P(splits.data_ptr()), st or sp)
        assert rc == 0, rc

    def call_attention(kv, st=None):
        rc = lib.mla_decode_attention(P(q.data_ptr()), P(kv.data_ptr()), P(bt.data_ptr()), P(sl.data_ptr()),
                                      B, s_q, H, kv.shape[0], bt.shape[1], ctypes.c_float(inp.scale), n_sms,
                                      P(sched.data_ptr()), P(splits.data_ptr()), P(ws.data_ptr()), ws_bytes,
                                      P(out.data_ptr()), P(lse.data_ptr()), st or sp)
        assert rc == 0, rc

    def call_combine(st=None):
        rc = lib.mla_decode_combine(P(splits.data_ptr()), P(sched.data_ptr()), P(ws.data_ptr()), ws_bytes,
                                    B, s_q, H, n_sms, P(out.data_ptr()), P(lse.data_ptr()), st or sp)
        assert rc == 0, rc

    # ---- warm-up (untimed)
    for k in range(max(3, args.warmup)):
        call_metadata(); call_attention(kv_copies[k % n_copies]); call_combine()
    torch.cuda.synchronize(dev)
    assert mla.get_device_error(sched) == 0

    # ---- accuracy against the fp64 oracle on sampled sequences (rank 0, N = 1)
    acc = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        call_metadata(); call_attention(kv_copies[0]); call_combine()
        torch.cuda.synchronize(dev)
        seqs = ACCURACY_SAMPLE.get(args.workload) if not args.batch else [0]
        r_out, r_lse = oracle.default().direct(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.scale,
                                               seqs=seqs)
        acc = accuracy(out.float().cpu().numpy(), lse.cpu().numpy(), r_out, r_lse, seqs, B)

    # ---- timed region 1: K steps, each on the other copy of the cache, with
    # an event between kernels to time each one
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    sampler = ClockSampler(local).start()
    time.sleep(0.3)
    barrier(dev)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    for k in range(K):
        e = ev[k]
        e[0].record(stream)
        call_metadata()
        e[1].record(stream)
        call_attention(kv_copies[k % n_copies])
        e[2].record(stream)
        call_combine()
        e[3].record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    meta_ms = [e[0].elapsed_time(e[1]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    comb_ms = [e[2].elapsed_time(e[3]) for e in ev]
    mean_attn_ms = max_over_ranks(statistics.mean(attn_ms), dev)

    # ---- timed region 2: K whole steps, events only around each step, so the
    # three launches run back to back as they would in serving
    ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(dev)
    torch.cuda.synchronize(dev)
    for k in range(K):
        e = ev2[k]
        e[0].record(stream)
        call_metadata()
        call_attention(kv_copies[k % n_copies])
        call_combine()
        e[1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    t_wall1 = time.time()
    clocks = sampler.stop(t_wall0, t_wall1)
    step_ms = [e[0].elapsed_time(e[1]) for e in ev2]
    mean_step_ms = max_over_ranks(statistics.mean(step_ms), dev)
    assert mla.get_device_error(sched) == 0

    # ---- timed region 3: attention + combine only, the schedule built once
    # (serving reuses it across the layers of a step)
    call_metadata()
    ev3 = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    torch.cuda.synchronize(dev)
    for k in range(K):
        e = ev3[k]
        e[0].record(stream)
        call_attention(kv_copies[k % n_copies])
        call_combine()
        e[1].record(stream)
    torch.cuda.synchronize(dev)
    amortised_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in ev3), dev)

    # ---- the same step replayed from a CUDA graph: one graph holds one step
    # per cache copy (up to 64), so consecutive steps still read different copies
    graph_steps = min(n_copies, 64)
    graph_us = None
    try:
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap):
            cp = ctypes.c_void_p(cap.cuda_stream)
            for k in range(graph_steps):
                call_metadata(cp); call_attention(kv_copies[k], cp); call_combine(cp)
        stream.wait_stream(cap)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(dev)
        reps = max(3, K // graph_steps)
        ga, gb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ga.record(stream)
        for _ in range(reps):
            g.replay()
        gb.record(stream)
        torch.cuda.synchronize(dev)
        graph_us = ga.elapsed_time(gb) / (reps * graph_steps) * 1e3
        del g
    except Exception as exc:  # capture is an extra figure; the step timing above stands
        print(f"cuda graph capture failed: {exc}", file=sys.stderr)
    if world > 1:
        graph_us = max_over_ranks(graph_us if graph_us is not None else float("nan"), dev)
    assert mla.get_device_error(sched) == 0

    # ---- end to end through the C ABI from pinned host memory: the step's
    # inputs (q, page table, lengths) sit back to back in one pinned buffer
    # and go over in one copy; out and lse come back in one copy.  The C ABI
    # takes the device addresses of the pieces.
    def pack(tensors, device):
        offs, total = [], 0
        for t in tensors:
            offs.append(total)
            total += (t.numel() * t.element_size() + 255) // 256 * 256
        buf = torch.empty(total, dtype=torch.uint8, device=device)
        views = [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for o, t in zip(offs, tensors)]
        return buf, views

    host_in, (q_h, bt_h, sl_h) = pack([inp.q, inp.block_table, inp.cache_seqlens], "cpu")
    q_h.copy_(inp.q); bt_h.copy_(inp.block_table); sl_h.copy_(inp.cache_seqlens)
    host_in = host_in.pin_memory()
    dev_in, (q, bt, sl) = pack([inp.q, inp.block_table, inp.cache_seqlens], dev)
    dev_out, (out, lse) = pack([out, lse], dev)
    host_out = torch.empty(dev_out.numel(), dtype=torch.uint8).pin_memory()
    h2d = host_in.numel()
    d2h = host_out.numel()
    K2 = max(10, K // 4)
    e2e_ms = []
    for k in range(K2 + 3):
        a = torch.cuda.Event(enable_timing=True)
        b_ = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dev_in.copy_(host_in, non_blocking=True)
        call_metadata(); call_attention(kv_copies[k % n_copies]); call_combine()
        host_out.copy_(dev_out, non_blocking=True)
        b_.record(stream)
        b_.synchronize()
        if k >= 3:
            e2e_ms.append(a.elapsed_time(b_))
    e2e_us = max_over_ranks(statistics.mean(e2e_ms), dev) * 1e3
    assert mla.get_device_error(sched) == 0

    # ---- roofline of the attention kernel
    alg_bytes = mi.algorithmic_bytes(inp)
    alg_flops = mi.algorithmic_flops(inp)
    roof = roofline(alg_bytes, alg_flops, mean_attn_ms * 1e-3, measured_peaks())
    t_attn = mean_attn_ms * 1e-3
    roof["both"]["hbm_frac_of_nominal_8tbs"] = alg_bytes / t_attn / 8e12
    roof["both"]["tensor_frac_of_sustained"] = alg_flops / t_attn / (sustained_tflops() * 1e12)
    roof["traffic"] = ncu_traffic(args.workload) if not args.batch else None
    roof["kernel"] = attention_kernel_name(s_q, H)
    roof["algorithmic_bytes_per_launch"] = alg_bytes
    roof["algorithmic_flops_per_launch"] = alg_flops

    line = {
        "metric": METRIC,
        "value": mean_step_ms * 1e3,
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": mean_step_ms,
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "B": B, "s_q": s_q, "H": H, "seqlen": w.seqlen,
                   "page": mi.PAGE, "table": w.table, "kv_bytes": int(inp.kv_cache.numel() * 2),
                   "l2": f"inputs larger than L2: {n_copies} device copies of the {kv_bytes / 2**20:.1f} MiB cache, used in turn step by step ({n_copies * kv_bytes / l2:.1f}x the {l2 >> 20} MiB L2); no flush",
                   "parallelism": f"replicas x{world} (independent batches)", "num_sms": n_sms},
        "kernels_us": {"metadata": statistics.mean(meta_ms) * 1e3, "attention": statistics.mean(attn_ms) * 1e3,
                       "combine": statistics.mean(comb_ms) * 1e3},
        "achieved_tb_s": alg_bytes / (mean_step_ms * 1e-3) / 1e12,
        "achieved_tflop_s": alg_flops / (mean_step_ms * 1e-3) / 1e12,
        "roofline": roof,
        "e2e": {"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "call_schedule_amortised_us": amortised_ms * 1e3,
        "cuda_graph_us": graph_us,
        "gpu_launches": 3 * K,  # per timed region
        "timing": ("value/ms_per_step: events around whole steps (region 2); kernels_us and roofline: events "
                   "between kernels (region 1); call_schedule_amortised_us: attention + combine with the schedule "
                   "built once (region 3); cuda_graph_us: whole steps replayed from a CUDA graph"),
        "clocks": clocks,
    }
    if acc is not None:
        line["accuracy"] = acc
    if world > 1:
        line["aggregate_calls_per_s"] = world / (mean_step_ms * 1e-3)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inp)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def run_context_parallel_rank(args):
    """One rank of a W-way context-parallel decode, on one GPU: the decode of
    this rank's 1/W of every sequence's pages (metadata + attention +
    combine), then the merge of W partial states.  The all-gather between
    them (W x B x H x 1028 bytes over NVLink) needs W GPUs and is not timed;
    its size is reported."""
    import ctypes

    import decode_attention_latent_b200 as mla
    from decode_attention_latent_b200.context_parallel import local_shard

    W = args.context_parallel
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    lib = mla.load_library()
    w = selected_workload(args)
    if w.s_q != 1:
        raise SystemExit("context-parallel decode takes s_q = 1 workloads")
    inp = mi.make_inputs(w, seed=0)
    B, H = w.B, w.H
    sl_h, bt_h = local_shard(inp.cache_seqlens, inp.block_table, W, 0)
    n_sms = mla.num_sms(dev)
    q = inp.q.to(dev)
    n_copies = kv_copy_count(int(sl_h.clamp(min=0).sum()) * 1152, L2_BYTES)
    kv_copies = [inp.kv_cache.to(dev) for _ in range(min(n_copies, 4))]
    bt, sl = bt_h.to(dev), sl_h.to(dev)
    sched = torch.empty(mla.sched_meta_ints(n_sms), dtype=torch.int32, device=dev)
    splits = torch.empty(B + 1, dtype=torch.int32, device=dev)
    ws_bytes = mla.workspace_size(B, 1, H, n_sms)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    parts = torch.zeros(W, B, 1, H, mi.D_V, dtype=torch.bfloat16, device=dev)
    lse_parts = torch.zeros(W, B, 1, H, dtype=torch.float32, device=dev)
    out = torch.empty(B, 1, H, mi.D_V, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, 1, H, dtype=torch.float32, device=dev)
    sp = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    P = ctypes.c_void_p

    def local_decode(kv):
        assert lib.mla_decode_metadata(P(sl.data_ptr()), B, 1, H, n_sms, P(sched.data_ptr()),
                                       P(splits.data_ptr()), sp) == 0
        assert lib.mla_decode(P(q.data_ptr()), P(kv.data_ptr()), P(bt.data_ptr()), P(sl.data_ptr()), B, 1, H,
                              kv.shape[0], bt.shape[1], ctypes.c_float(inp.scale), n_sms, P(sched.data_ptr()),
                              P(splits.data_ptr()), P(ws.data_ptr()), ws_bytes, P(parts[0].data_ptr()),
                              P(lse_parts[0].data_ptr()), sp) == 0

    def merge():
        assert lib.mla_merge_states(P(parts.data_ptr()), P(lse_parts.data_ptr()), W, B * H, P(out.data_ptr()),
                                    P(lse.data_ptr()), sp) == 0

    for k in range(max(3, args.warmup)):
        local_decode(kv_copies[k % len(kv_copies)])
    parts[1:] = parts[0]
    lse_parts[1:] = lse_parts[0]
    for _ in range(max(3, args.warmup)):
        merge()
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    ev[0].record()
    for k in range(args.steps):
        local_decode(kv_copies[k % len(kv_copies)])
    ev[1].record()
    ev[2].record()
    for _ in range(args.steps):
        merge()
    ev[3].record()
    torch.cuda.synchronize(dev)
    assert mla.get_device_error(sched) == 0
    dec_us = ev[0].elapsed_time(ev[1]) * 1e3 / args.steps
    mer_us = ev[2].elapsed_time(ev[3]) * 1e3 / args.steps
    shard_tokens = int(sl_h.sum())
    line = {
        "metric": "MLA context-parallel decode us/call per rank (one rank of a W-way length split)",
        "value": dec_us + mer_us, "unit": "us/call", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": False, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "W": W, "B": B, "H": H, "shard_tokens_rank0": shard_tokens,
                   "full_tokens": int(inp.cache_seqlens.sum()), "kv_copies": len(kv_copies)},
        "decode_us": dec_us, "merge_us": mer_us,
        "gather_bytes_per_rank": W * B * H * (mi.D_V * 2 + 4),
        "not_timed": "the all-gather of the W states: one GPU emulates one rank",
    }
    print(json.dumps(line))
    return 0


def run_fp8(args):
    """The decode over an FP8 (e4m3, one fp32 scale per token) cache of the same
    workload (16 or 32 query columns), one GPU: per call the metadata, attention and combine kernels
    (as the default line), the attention kernel alone and its roofline on
    576 + 4 bytes per cached token, and the error against the oracle's FP8
    definition."""
    import ctypes

    import decode_attention_latent_b200 as mla

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    lib = mla.load_library()
    w = selected_workload(args)
    if w.s_q * w.H not in (16, 32) or w.s_q > 2:
        raise SystemExit("the FP8 cache path takes 16 or 32 query columns (H = 16 with s_q <= 2, or H = 32)")
    inp = mi.make_inputs(w, seed=0)
    nb = inp.kv_cache.shape[0]
    inp.kv_cache = None  # the bf16 cache is not used here
    cache = mi.fp8_cache(nb, seed=1)
    B, S, H = w.B, w.s_q, w.H
    n_sms = mla.num_sms(dev)
    fp8_bytes = nb * 64 * (576 + 4)
    n_copies = kv_copy_count(fp8_bytes, L2_BYTES)
    codes = [cache.codes.to(dev) for _ in range(n_copies)]
    scales = [cache.scale.to(dev) for _ in range(n_copies)]
    q, bt, sl = inp.q.to(dev), inp.block_table.to(dev), inp.cache_seqlens.to(dev)
    sched = torch.empty(mla.sched_meta_ints(n_sms), dtype=torch.int32, device=dev)
    splits = torch.empty(B + 1, dtype=torch.int32, device=dev)
    ws_bytes = mla.workspace_size(B, S, H, n_sms)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.empty(B, S, H, mi.D_V, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, S, H, dtype=torch.float32, device=dev)
    sp = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    P = ctypes.c_void_p

    def meta():
        assert lib.mla_decode_metadata(P(sl.data_ptr()), B, S, H, n_sms, P(sched.data_ptr()),
                                       P(splits.data_ptr()), sp) == 0

    def decode(k, fn):
        c, s_ = codes[k % n_copies], scales[k % n_copies]
        assert fn(P(q.data_ptr()), P(c.data_ptr()), P(s_.data_ptr()), P(bt.data_ptr()),
                  P(sl.data_ptr()), B, S, H, nb, bt.shape[1], ctypes.c_float(inp.scale),
                  n_sms, P(sched.data_ptr()), P(splits.data_ptr()), P(ws.data_ptr()),
                  ws_bytes, P(out.data_ptr()), P(lse.data_ptr()), sp) == 0

    def call(k):
        meta()
        decode(k, lib.mla_decode_fp8)

    for k in range(max(3, args.warmup)):
        call(k)
    torch.cuda.synchronize(dev)
    acc = None
    if not args.no_cpu_baseline:
        import oracle
        call(0)
        torch.cuda.synchronize(dev)
        r_out, r_lse = oracle.default().direct_fp8(inp.q, cache.codes, cache.scale, inp.block_table,
                                                   inp.cache_seqlens, inp.scale)
        acc = accuracy(out.float().cpu().numpy(), lse.cpu().numpy(), r_out, r_lse, None, B)
    sampler = ClockSampler(0).start()
    time.sleep(0.3)
    t_start = time.time()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for k in range(args.steps):
        ev[k][0].record(); call(k); ev[k][1].record()
    torch.cuda.synchronize(dev)
    assert mla.get_device_error(sched) == 0
    call_us = statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e3
    meta()
    ea = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for k in range(args.steps):
        ea[k][0].record(); decode(k, lib.mla_decode_attention_fp8); ea[k][1].record()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop(t_start, time.time())
    assert mla.get_device_error(sched) == 0
    attn_us = statistics.mean(a.elapsed_time(b) for a, b in ea) * 1e3
    tokens = int(inp.cache_seqlens.sum())
    alg = tokens * (576 + 4) + q.numel() * 2 + out.numel() * 2 + lse.numel() * 4 + sum(
        (int(L) + 63) // 64 for L in inp.cache_seqlens.tolist()) * 4 + B * 4
    hbm = measured_peaks()[0]
    traffic = None
    path = os.path.join(ROOT, "profiles", f"mla_decode_fp8_{args.workload}.md")
    if os.path.exists(path) and not args.batch:
        text = open(path).read()
        m_b = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
        m_s = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
        if m_b and m_s and m_s.group(1) == source_digest():
            traffic = float(m_b.group(1))
    line = {
        "metric": "MLA decode us/call over an FP8 (e4m3, per-token scale) cache", "value": call_us, "unit": "us/call",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": False,
        "dtype": "e4m3 cache and e4m3 MMA operands (q, weights as two e4m3 terms), fp32 accumulate",
        "data": "synthetic",
        "config": {"workload": args.workload, "B": B, "s_q": S, "H": H, "cache_copies": n_copies},
        "attention_us": attn_us,
        "roofline": {"bound": "hbm", "achieved": alg / (attn_us * 1e-6) / 1e9, "peak": hbm, "unit": "GB/s",
                     "frac": alg / (attn_us * 1e-6) / 1e9 / hbm, "algorithmic_bytes_per_launch": alg,
                     "traffic": traffic, "kernel": f"mla_decode_kernel<{S * H},{S},true>"},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    if acc is not None:
        line["accuracy"] = acc
    print(json.dumps(line))
    return 0


def run_naive(args):
    """The non-absorbed form (mla_decode_naive) on the workload's cache, one
    GPU: per-head up-projections of every tile on the tensor cores, so the
    roofline is the bf16 tensor peak over its algorithmic FLOPs; the error
    against the oracle's non-absorbed form on a bounded sample (the fp64
    decompression of every token is too slow for the whole workload)."""
    import numpy as np

    import decode_attention_latent_b200 as mla

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    mla.load_library()
    w = selected_workload(args)
    if w.s_q > 2:
        raise SystemExit("the non-absorbed form takes s_q <= 2")
    inp = mi.make_inputs(w, seed=0)
    nv = mi.naive_inputs(w.B, w.s_q, w.H, seed=1)
    q, kv, wk, wv = nv.q.to(dev), inp.kv_cache.to(dev), nv.w_uk.to(dev), nv.w_uv.to(dev)
    bt, sl = inp.block_table.to(dev), inp.cache_seqlens.to(dev)
    out, lse, err = mla.decode_naive(q, kv, wk, wv, bt, sl, inp.scale)
    for _ in range(max(3, args.warmup)):
        mla.decode_naive(q, kv, wk, wv, bt, sl, inp.scale, out=out, lse=lse, error_word=err)
    torch.cuda.synchronize(dev)
    assert int(err.item()) == 0
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(0).start()
    time.sleep(0.3)
    t0 = time.time()
    for k in range(K):
        ev[k][0].record(); mla.decode_naive(q, kv, wk, wv, bt, sl, inp.scale, out=out, lse=lse, error_word=err)
        ev[k][1].record()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop(t0, time.time())
    assert int(err.item()) == 0
    call_us = statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e3
    flops = mi.naive_algorithmic_flops(inp)
    _, _, tc, tc_src = measured_peaks()
    achieved = flops / (call_us * 1e-6) / 1e12
    acc = None
    if not args.no_cpu_baseline:
        import oracle
        # bounded sample: the first two sequences cut to 1024 tokens, same q and matrices
        sub = mi.Inputs(q=inp.q[:2], kv_cache=inp.kv_cache, block_table=inp.block_table[:2],
                        cache_seqlens=inp.cache_seqlens[:2].clamp(max=1024), scale=inp.scale)
        g_out, g_lse, _ = mla.decode_naive(q[:2].contiguous(), kv, wk, wv, bt[:2].contiguous(),
                                           sub.cache_seqlens.to(dev), inp.scale)
        torch.cuda.synchronize(dev)
        r_out, r_lse = oracle.default().naive(nv.q[:2], inp.kv_cache, nv.w_uk, nv.w_uv, sub.block_table,
                                              sub.cache_seqlens, inp.scale)
        acc = accuracy(g_out.float().cpu().numpy(), g_lse.cpu().numpy(), r_out, r_lse, None, 2)
        acc["sequences"] = "2 sequences cut to their first 1024 tokens"
    line = {
        "metric": "MLA decode, non-absorbed form (per-tile up-projection) us/call", "value": call_us,
        "unit": "us/call", "n_gpus": 1, "steps": K, "warmup": args.warmup, "higher_is_better": False,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "B": w.B, "s_q": w.s_q, "H": w.H, "kv_bytes": int(inp.kv_cache.numel() * 2),
                   "weights": "w_uk, w_uv [H, 128, 512] bf16, N(0, 1/512)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": tc, "unit": "TFLOP/s", "frac": achieved / tc,
                     "peak_source": tc_src, "frac_of_sustained": achieved / sustained_tflops(),
                     "algorithmic_flops_per_launch": flops, "traffic": None,
                     "kernel": f"mla_naive_kernel<{w.s_q}>"},
        "gpu_launches": 2 * K,
        "clocks": clocks,
    }
    if acc is not None:
        line["accuracy"] = acc
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=mi.HEADLINE, choices=sorted(mi.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0,
                    help="cut the workload to its first BATCH sequences (profiler captures on a smaller case)")
    ap.add_argument("--fp8", action="store_true", help="the same workload over an FP8 (e4m3) cache (H = 16, s_q = 1)")
    ap.add_argument("--naive", action="store_true",
                    help="the non-absorbed form (per-tile up-projection) on the same workload")
    ap.add_argument("--context-parallel", type=int, default=0, metavar="W",
                    help="time one rank of a W-way context-parallel decode on one GPU (s_q = 1 workloads)")
    args = ap.parse_args(argv)
    world, rank, local = dist_env()
    if args.context_parallel >= 2 and args.impl == "ours":
        return run_context_parallel_rank(args)
    if args.fp8 and args.impl == "ours":
        return run_fp8(args)
    if args.naive and args.impl == "ours":
        return run_naive(args)
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_ours(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
