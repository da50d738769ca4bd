#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200 through libkda's C ABI.

A *step* is one pass of the prefill hot path over the K3-layer-shaped
workload: ``kda_prologue`` (short conv + SiLU + L2 over 32768 tokens x 96
heads x 128 channels of q/k/v projections, fp16 q/k/v out) followed by
``kda_chunk_fwd`` (tensor-core chunkwise prefill, chunk 64, fp32 state) with a
preallocated workspace: its two-pass form, a parallel prep pass over every
(chunk, head) and a state pass over (sequence, head, value slice).  The
one-pass chunk kernel and the fused variant ``kda_prologue_chunk_fwd`` are
timed beside it.  ``value`` is prefill tokens/s
(a token is one position through all 96 heads) with inputs resident in HBM.
The batched decode step (256 sequences x 96 heads, 100 consecutive steps,
state updated in place) is timed in the same run and reported under
``decode``.

Usage: ``python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]``.
With N > 1 launch one process per GPU (torchrun); every rank runs its own
replica of the workload (the problems are independent: no collective on the
data path) and the slowest rank's time is reported.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import resource
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "KDA prefill tokens/s & decode tokens/s at H=96,d=128 on 1 B200; % of roofline"
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0

# Algorithmic work per token-head (d = 128; see the design notes).
D_ = 128
QKV_DT = 2                                          # q/k/v handed from prologue to chunk: f16
PROLOGUE_BYTES_PER_TH = 3 * D_ * 2 + 3 * D_ * QKV_DT   # read x (bf16), write q/k/v      = 1536
# The algorithmic bytes of the chunk call as first planned: q, k, v (16-bit) + g + beta
# + o in the activation type (16-bit) = 1540 per token-head.  The library writes o in
# fp32 (its read-out is heavy-tailed: a 16-bit o alone breaks the parity bound), which
# makes 1796; both fractions are reported.
CHUNK_BYTES_PER_TH_PLAN = 3 * D_ * QKV_DT + D_ * 4 + 4 + D_ * 2
CHUNK_BYTES_PER_TH = 3 * D_ * QKV_DT + D_ * 4 + 4 + D_ * 4  # q,k,v + g + beta + o (f32) = 1796
FUSED_BYTES_PER_TH = 3 * D_ * 2 + D_ * 4 + 4 + D_ * 4  # x + g + beta + o: the fused floor = 1796
GATED_BYTES_PER_TH = 3 * D_ * 2 + D_ * 2 + 4 + D_ * 4  # bf16 q,k,v + bf16 g_raw + beta + o = 1540
EPILOGUE_BYTES_PER_TH = D_ * 4 + 2 * D_ * 2             # o (f32) + gate, out (bf16) = 1024
# backward: q, k, v (fp16) + g + beta + dL/do in; dq, dk, dv, dg (f32) + dbeta out = 3848
BWD_BYTES_PER_TH = 3 * D_ * 2 + D_ * 4 + 4 + D_ * 4 + 4 * D_ * 4 + 4
CHUNK_FLOPS_PER_TH = 139392                        # chunk form, d=128, C=64
# decode per (sequence, head): state read+write, x, conv cache read+write, g, beta, o (f32)
DECODE_BYTES_PER_SH = 2 * D_ * D_ * 4 + 3 * D_ * 2 + 2 * 3 * 3 * D_ * 2 + D_ * 4 + 4 + D_ * 4

_CSRC = "gated_delta_rule_prologue_b200/csrc/"
# the device headers every kernel file includes
_HDRS = [_CSRC + "kda_common.cuh", _CSRC + "kda_tcgen05.cuh", _CSRC + "kda_chunk_record.cuh"]
KERNEL_SOURCES = {
    "kda_prologue_chunk_fwd": [_CSRC + "kda_chunk_tc.cu", _CSRC + "kda_chunk_state.cu"] + _HDRS,
    "kda_prologue_chunk_fwd_one_pass": [_CSRC + "kda_chunk_tc.cu"] + _HDRS,
    "kda_prologue": [_CSRC + "kda_prologue.cu"] + _HDRS,
    "kda_chunk_fwd": [_CSRC + "kda_chunk_tc.cu", _CSRC + "kda_chunk_state.cu"] + _HDRS,
    "kda_chunk_fwd_one_pass": [_CSRC + "kda_chunk_tc.cu"] + _HDRS,
    "kda_chunk_fwd_gated": [_CSRC + "kda_chunk_tc.cu", _CSRC + "kda_chunk_state.cu"] + _HDRS,
    "kda_output_epilogue": [_CSRC + "kda_epilogue.cu"] + _HDRS,
    "kda_chunk_bwd": [_CSRC + "kda_chunk_tc.cu", _CSRC + "kda_chunk_state.cu",
                      _CSRC + "kda_chunk_bwd.cu"] + _HDRS,
    "kda_decode_step": [_CSRC + "kda_decode.cu"] + _HDRS,
    "kda_chunk_fwd_windowed64": [_CSRC + "kda_chunk_tc.cu", _CSRC + "kda_chunk_state.cu"] + _HDRS,
}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(
            p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def src_sha(rels):
    """sha256 (first 16 hex digits) of the concatenated sources of one call."""
    h = hashlib.sha256()
    for rel in rels:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per call from the committed ncu summary (summed over the
    call's launches), if it was taken on the current sources (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    sha = src_sha(KERNEL_SOURCES[kernel])
    for line in open(path):
        if line.startswith("#") or "=" not in line:
            continue
        kv = dict(tok.split("=", 1) for tok in line.split() if "=" in tok)
        if kv.get("kernel") == kernel and kv.get("src_sha256") == sha:
            return float(kv["dram_bytes_per_launch"])
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.rows = []
        self.sel = []
        try:
            props = torch.cuda.get_device_properties(device)
            uuid = getattr(props, "uuid", None)
            if uuid is not None:
                u = str(uuid)
                self.sel = ["-i", u if u.startswith("GPU-") else "GPU-" + u]
        except Exception:
            self.sel = []

    def start(self):
        self.tmp = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *self.sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        sm, mx, reasons = [], [], set()
        for line in self.tmp.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        os.unlink(self.tmp.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=300),
            device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x, world):
    """The largest of the ranks' values (device timings are compared on every
    rank; the slowest rank defines the job's time)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank, local_ms):
    """Whole-job units/s for replicas that each process `units_per_rank` units:
    every rank's units over the slowest rank's time.  Returns (value, max_ms)."""
    ms = max_over_ranks(local_ms, world)
    return world * units_per_rank / (ms * 1e-3), ms


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def roofline(bound, algo, ms, peak, unit, traffic):
    achieved = algo / (ms * 1e-3) / (1e9 if unit == "GB/s" else 1e12)
    return {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": traffic}


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(n_tokens):
    """The float64 oracle on the first ``n_tokens`` tokens of the K3-layer
    workload, all 96 heads (prologue + recurrence).  Returns (seconds, cores)."""
    import numpy as np
    from oracle import kda_recurrent, prologue
    c = W.WORKLOADS["k3_prefill"]
    H, D = c["H"], c["D"]
    heads = [W.k3_prefill_head(h, T=n_tokens) for h in range(H)]
    x = torch.stack([hh[0] for hh in heads], dim=2).reshape(n_tokens, 3 * H * D)
    w = torch.stack([hh[1] for hh in heads], dim=1).reshape(3 * H * D, 4)
    g = torch.stack([hh[2] for hh in heads], dim=1)
    beta = torch.stack([hh[3] for hh in heads], dim=1)
    r0 = resource.getrusage(resource.RUSAGE_SELF)
    t0 = time.perf_counter()
    q, k, v, _ = prologue(x, w, H, D)
    o, _ = kda_recurrent(q, k, v, g, beta, 1.0)
    wall = time.perf_counter() - t0
    r1 = resource.getrusage(resource.RUSAGE_SELF)
    cpu = (r1.ru_utime - r0.ru_utime) + (r1.ru_stime - r0.ru_stime)
    assert np.all(np.isfinite(o))
    return wall, max(1, round(cpu / wall))


# Tokens of the K3-layer workload (all 96 heads) the oracle runs per sample, in the
# cpu_baseline leg and in every step of the reference arm alike.
ORACLE_SAMPLE_TOKENS = 768
ORACLE_NOTE = ("the oracle is single-threaded by construction: a Python loop over tokens "
               "with float64 NumPy vectorised over heads, so BLAS threading does not engage")


def cpu_baseline(n_tokens=ORACLE_SAMPLE_TOKENS):
    wall, cores = oracle_sample(n_tokens)
    return {"value": round(n_tokens / wall, 3), "unit": "tokens/s", "cores": cores,
            "host_cores_available": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"first {n_tokens} tokens of the K3-layer prefill, all 96 heads "
                      f"(prologue + token-by-token recurrence, float64 NumPy), {wall:.1f} s",
            "note": ORACLE_NOTE}


# Bytes of one record of the two-pass prefill and the workspace of one K3 call (the
# library's layout: a 1 KiB index header, then (ceil(T/64) + 1) * H records).
RECORD_BYTES = 90880


def k3_config(world, T=32768, H=96, D=128):
    """The benchmark's workload description, shared by both arms."""
    th = T * H
    ws_bytes = 1024 + ((T + 63) // 64 + 1) * H * RECORD_BYTES
    step_gb = (PROLOGUE_BYTES_PER_TH * th + CHUNK_BYTES_PER_TH * th + 2 * ws_bytes) / 1e9
    return {
        "workload": "k3_prefill: kda_prologue (fp16 q/k/v out) + kda_chunk_fwd (two-pass, "
                    "preallocated workspace) over T=32768 tokens, H=96, d_k=d_v=128, "
                    "chunk 64, bf16 q/k/v projections, fp32 g/beta/state/o",
        "global_batch": world, "seq_len": T, "heads": H, "head_dim": D,
        "parallelism": f"replicas x{world} (independent problems, no collective)",
        "l2": f"inputs larger than L2 ({step_gb:.1f} GB touched per step, no flush needed)",
    }


def run_reference(args, world, rank):
    if rank != 0:
        return
    # the same sample as the cpu_baseline leg, shrunk only if the run would exceed ~5 min
    budget_s = 300.0
    per_token_s = 0.011
    n_tok = int(max(16, min(ORACLE_SAMPLE_TOKENS,
                            budget_s / max(1, args.steps + args.warmup) / per_token_s)))
    for _ in range(args.warmup):
        oracle_sample(n_tok)
    times, cores = [], 1
    for _ in range(args.steps):
        wall, cores = oracle_sample(n_tok)
        times.append(wall)
    ms = 1e3 * statistics.mean(times)
    value = n_tok / (ms * 1e-3)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": k3_config(world),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"first {n_tok} tokens x 96 heads of the K3-layer prefill "
                                   "per step (prologue + recurrence, float64)",
                         "note": ORACLE_NOTE},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def seq4k_side(kda, dev, stream, hbm):
    """The single-sequence bf16 prefill (T=4096, H=8, d=128, initial state):
    its 32 (head, value slice) chains fill a fifth of the GPU, so the library
    splits the sequence into segments (sequence-parallel state pass).  Timed
    split and whole, L2 flushed before every call (the inputs fit in L2)."""
    sinp = W.seq4k_bf16()
    T4, H4, D4 = sinp.T, sinp.H, sinp.q.shape[2]
    q4, k4, v4 = sinp.q.to(dev), sinp.k.to(dev), sinp.v.to(dev)
    g4, b4, s04 = sinp.g.to(dev), sinp.beta.to(dev), sinp.initial_state.to(dev)
    o4 = torch.empty((T4, H4, D4), dtype=torch.float32, device=dev)
    f4 = torch.empty_like(s04)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    L = kda.kda_chunk_fwd_segment_chunks(1, T4, H4)
    out = {"workload": "seq4k_bf16: T=4096, H=8, d_k=d_v=128, chunk 64, bf16 q/k/v, "
                       "initial state, one sequence", "segment_chunks": L,
           "l2": "256 MiB written before every timed call"}
    for name, seg in (("split", None), ("whole", 0)):
        nb = (kda.kda_chunk_fwd_workspace_bytes(1, T4, H4, D4, D4, 64, q4.dtype) if seg is None
              else kda.kda_chunk_fwd_segmented_workspace_bytes(1, T4, H4, D4, D4, 64, q4.dtype,
                                                               seg))
        ws4 = torch.empty(nb, dtype=torch.uint8, device=dev)
        call = lambda: kda.kda_chunk_fwd(q4, k4, v4, g4, b4, o4, scale=sinp.scale,
                                         initial_state=s04, final_state=f4, workspace=ws4,
                                         segment_chunks=seg, stream=stream)
        for _ in range(3):
            call()
        times = []
        for _ in range(10):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        out[name] = dict(ms=round(ms, 4), tokens_per_s=round(T4 / (ms * 1e-3), 1),
                         **roofline("hbm", CHUNK_BYTES_PER_TH * T4 * H4, ms, hbm, "GB/s", None))
        del ws4
    assert kda.kda_get_device_status() == 0
    out["speedup"] = round(out["whole"]["ms"] / out["split"]["ms"], 3)
    del q4, k4, v4, g4, b4, s04, o4, f4, flush
    return out


def varlen_side(kda, dev, stream, hbm):
    """The packed varlen prefill: 16 sequences of uniform length in [512, 16384]
    (93,891 tokens as drawn), H=32, d=128, bf16 q/k/v, an initial state per
    sequence and every final state returned, through kda_chunk_fwd with
    cu_seqlens and a preallocated workspace.  Its inputs are larger than L2."""
    vinp = W.varlen16()
    Tv, Hv, Dv, Nv = vinp.T, vinp.H, vinp.q.shape[2], vinp.N
    qv, kv, vv = vinp.q.to(dev), vinp.k.to(dev), vinp.v.to(dev)
    gv, bv, s0v = vinp.g.to(dev), vinp.beta.to(dev), vinp.initial_state.to(dev)
    cu = vinp.cu_seqlens.to(dev)
    ov = torch.empty((Tv, Hv, Dv), dtype=torch.float32, device=dev)
    fv = torch.empty_like(s0v)
    wsv = torch.empty(kda.kda_chunk_fwd_workspace_bytes(Nv, Tv, Hv, Dv, Dv, 64, qv.dtype),
                      dtype=torch.uint8, device=dev)
    call = lambda: kda.kda_chunk_fwd(qv, kv, vv, gv, bv, ov, scale=vinp.scale,
                                     initial_state=s0v, final_state=fv, cu_seqlens=cu,
                                     workspace=wsv, stream=stream)
    for _ in range(3):
        call()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(5)]
    for e in ev:
        e[0].record(stream)
        call()
        e[1].record(stream)
    torch.cuda.synchronize(dev)
    assert kda.kda_get_device_status() == 0
    ms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    th = Tv * Hv
    states = 2 * Nv * Hv * Dv * Dv * 4  # initial state read, final state written
    out = {"workload": f"varlen16: {Nv} packed sequences, {Tv} tokens (lengths uniform in "
                       f"[512, 16384]), H={Hv}, d=128, bf16 q/k/v, initial and final state "
                       "per sequence", "ms": round(ms, 4),
           "tokens_per_s": round(Tv / (ms * 1e-3), 1),
           "segment_chunks": kda.kda_chunk_fwd_segment_chunks(Nv, Tv, Hv),
           "roofline": dict(roofline("hbm", CHUNK_BYTES_PER_TH_PLAN * th + states, ms, hbm,
                                     "GB/s", None),
                            algorithmic_bytes=f"{CHUNK_BYTES_PER_TH_PLAN} B per token-head + "
                                              "the states (2 x 64 KiB per sequence-head)",
                            frac_fp32_readout_bytes=roofline(
                                "hbm", CHUNK_BYTES_PER_TH * th + states, ms, hbm, "GB/s",
                                None)["frac"])}
    del qv, kv, vv, gv, bv, s0v, cu, ov, fv, wsv
    return out


def tiny_side(kda, dev, stream):
    """The tiny fp32 forward (T=64, H=2, d=16, chunk 16: the exact-fp32 CUDA-core
    path): latency of one kda_chunk_fwd call, median over 200 calls."""
    t = W.tiny_f32()
    args_ = [x.to(dev) for x in (t.q, t.k, t.v, t.g, t.beta)]
    o = torch.empty(t.v.shape, dtype=torch.float32, device=dev)
    fs = torch.empty((1, t.H, t.q.shape[2], t.q.shape[2]), device=dev)
    call = lambda: kda.kda_chunk_fwd(*args_, o, scale=t.scale, final_state=fs, chunk=t.chunk,
                                     stream=stream)
    for _ in range(10):
        call()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(200)]
    for e in ev:
        e[0].record(stream)
        call()
        e[1].record(stream)
    torch.cuda.synchronize(dev)
    assert kda.kda_get_device_status() == 0
    us = 1e3 * statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    return {"workload": "tiny_f32: T=64, H=2, d_k=d_v=16, chunk 16, fp32 (CUDA-core path)",
            "latency_us": round(us, 2), "tokens_per_s": round(t.T / (us * 1e-6), 1)}


def decode_parity(state, cache, outs_last, steps, ns):
    """The oracle's run of the same ``steps`` decode steps on sequences ``ns``
    (all 96 heads), against the GPU's state, cache and last read-out."""
    import numpy as np
    from oracle import kda_decode_step, state_from_abi, state_to_abi
    st0, c0, xs, gs, bs, wr = W.decode256_seqs(ns, steps)
    c = W.WORKLOADS["decode256"]
    H, D = c["H"], c["D"]
    S, cc = state_from_abi(st0), c0
    t0 = time.perf_counter()
    for i in range(steps):
        o_ref, S, cc = kda_decode_step(xs[i], wr, cc, gs[i], bs[i], S, H, D)
    wall = time.perf_counter() - t0
    got_o = outs_last[ns].double().cpu().numpy()
    got_s = state[ns].double().cpu().numpy()
    rel_o = float(np.max(np.abs(got_o - o_ref)) / np.sqrt(np.mean(o_ref ** 2)))
    ref_s = state_to_abi(S)
    rel_s = float(np.linalg.norm(got_s - ref_s) / np.linalg.norm(ref_s))
    cache_ok = bool(np.array_equal(cache[ns].double().cpu().numpy(), cc))
    return {"sequences": list(ns), "heads": H, "steps": steps,
            "o_rel_max": round(rel_o, 6), "state_rel_fro": round(rel_s, 6),
            "cache_exact": cache_ok, "ok": bool(rel_o <= 2e-2 and rel_s <= 1e-2 and cache_ok),
            "bounds": "max|o - o_ref| / RMS(o_ref) <= 2e-2 (last step); "
                      "||S - S_ref||_F / ||S_ref||_F <= 1e-2",
            "oracle_s": round(wall, 1)}


def run_ours(args, world, rank, local):
    import gated_delta_rule_prologue_b200 as kda
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hbm, bf16_burst, bf16_sust, peak_kind = peaks()

    # ---- prefill workload (inputs resident in HBM) ----
    inp = W.k3_prefill(pin_memory=True)
    T, H, D = inp.T, inp.H, inp.D
    x = inp.x.to(dev)
    w = inp.conv_w.to(dev)
    g = inp.g.to(dev)
    beta = inp.beta.to(dev)
    o = torch.empty((T, H, D), dtype=torch.float32, device=dev)
    fs = torch.empty((1, H, D, D), dtype=torch.float32, device=dev)
    q = torch.empty((T, H, D), dtype=torch.float16, device=dev)
    k, v = torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(kda.kda_chunk_fwd_workspace_bytes(1, T, H, D, D, inp.chunk, q.dtype),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        kda.kda_prologue(x, w, q, k, v, H=H, D=D, stream=stream)
        kda.kda_chunk_fwd(q, k, v, g, beta, o, scale=inp.scale, final_state=fs,
                          chunk=inp.chunk, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert kda.kda_get_device_status() == 0
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        kda.kda_prologue(x, w, q, k, v, H=H, D=D, stream=stream)
        ev[i][1].record(stream)
        kda.kda_chunk_fwd(q, k, v, g, beta, o, scale=inp.scale, final_state=fs,
                          chunk=inp.chunk, workspace=ws, stream=stream)
        ev[i][2].record(stream)
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    value, ms_step = job_throughput(world, T, start.elapsed_time(end) / args.steps)
    pro_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    chk_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    assert kda.kda_get_device_status() == 0
    launches = 3 * args.steps  # prologue, chunk prep pass, chunk state pass

    # timed beside the step: the prologue fused into the two-pass chunk call, the
    # fused one-pass kernel, and the one-pass chunk kernel
    o2 = torch.empty_like(o)
    side = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(3)]
    for i in range(3):
        side[i][0].record(stream)
        kda.kda_prologue_chunk_fwd(x, w, g, beta, o2, H=H, D=D, scale=inp.scale, workspace=ws,
                                   stream=stream)
        side[i][1].record(stream)
        kda.kda_prologue_chunk_fwd(x, w, g, beta, o2, H=H, D=D, scale=inp.scale, workspace=None,
                                   stream=stream)
        side[i][2].record(stream)
        side[i][3].record(stream)
        kda.kda_chunk_fwd(q, k, v, g, beta, o2, scale=inp.scale, chunk=inp.chunk,
                          workspace=None, stream=stream)
        side[i][4].record(stream)
    torch.cuda.synchronize(dev)
    fused_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in side[1:])
    fused_one_pass_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in side[1:])
    one_pass_ms = statistics.mean(e[3].elapsed_time(e[4]) for e in side[1:])
    # the in-kernel gate: 16-bit gate pre-activations instead of the fp32 log-decay
    gen = torch.Generator().manual_seed(7)
    g_raw = torch.randn((T, H, D), generator=gen).to(torch.bfloat16).to(dev)
    A_log = (0.5 * torch.randn((H,), generator=gen)).to(dev)
    dt_bias = torch.randn((H, D), generator=gen).to(dev)
    gq = q.to(torch.bfloat16)
    gk, gv = k.to(torch.bfloat16), v.to(torch.bfloat16)
    gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(3)]
    for i in range(3):
        gev[i][0].record(stream)
        kda.kda_chunk_fwd_gated(gq, gk, gv, g_raw, beta, o2, A_log=A_log, dt_bias=dt_bias,
                                scale=inp.scale, workspace=ws, stream=stream)
        gev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    gated_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in gev[1:])
    # the windowed call: 64-chunk windows, a workspace that does not grow with T
    win_chunks = 64
    win_ws = torch.empty(kda.kda_chunk_fwd_windowed_workspace_bytes(1, T, H, D, D, inp.chunk,
                                                                    q.dtype, win_chunks),
                         dtype=torch.uint8, device=dev)
    wev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(3)]
    for i in range(3):
        wev[i][0].record(stream)
        kda.kda_chunk_fwd(q, k, v, g, beta, o2, scale=inp.scale, chunk=inp.chunk,
                          window_chunks=win_chunks, workspace=win_ws, stream=stream)
        wev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    windowed_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in wev[1:])
    win_ws_gb = win_ws.numel() / 1e9
    del win_ws
    # the output epilogue on the step's read-out (RMSNorm x sigmoid gate, bf16 out)
    ep_out = gq  # reuse a bf16 [T, H, D] buffer
    ep_w = (0.5 + torch.rand((D,), generator=gen)).to(dev)
    eev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(3)]
    for i in range(3):
        eev[i][0].record(stream)
        kda.kda_output_epilogue(o, g_raw, ep_w, ep_out, stream=stream)
        eev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    epi_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in eev[1:])
    del o2, g_raw, gq, gk, gv, ep_out
    # the prefill backward on the step's q/k/v (fp16), g, beta: dL/do ~ N(0,1) fp32
    d_o = torch.randn((T, H, D), generator=gen).to(dev)
    bwd_out = [torch.empty((T, H, D), device=dev) for _ in range(4)]
    d_beta = torch.empty((T, H), device=dev)
    bws = torch.empty(kda.kda_chunk_bwd_workspace_bytes(1, T, H, D, D, inp.chunk, q.dtype),
                      dtype=torch.uint8, device=dev)
    bev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(3)]
    for i in range(3):
        bev[i][0].record(stream)
        kda.kda_chunk_bwd(q, k, v, g, beta, d_o, scale=inp.scale, dq=bwd_out[0], dk=bwd_out[1],
                          dv=bwd_out[2], dg=bwd_out[3], dbeta=d_beta, want_d_initial_state=False,
                          workspace=bws, stream=stream)
        bev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    assert kda.kda_get_device_status() == 0
    bwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in bev[1:])
    del d_o, bwd_out, d_beta, bws
    torch.cuda.empty_cache()
    seq4k = seq4k_side(kda, dev, stream, hbm)
    varlen = varlen_side(kda, dev, stream, hbm)
    torch.cuda.empty_cache()
    tiny = tiny_side(kda, dev, stream)

    th = T * H
    # the shared workload description assumes the library's record layout
    assert ws.numel() == 1024 + ((T + 63) // 64 + 1) * H * RECORD_BYTES
    kernels = {
        "kda_prologue_chunk_fwd": dict(ms=round(fused_ms, 4), launches=2, **roofline(
            "hbm", FUSED_BYTES_PER_TH * th, fused_ms, hbm, "GB/s",
            recorded_traffic("kda_prologue_chunk_fwd"))),
        "kda_prologue_chunk_fwd_one_pass": dict(ms=round(fused_one_pass_ms, 4), **roofline(
            "hbm", FUSED_BYTES_PER_TH * th, fused_one_pass_ms, hbm, "GB/s",
            recorded_traffic("kda_prologue_chunk_fwd_one_pass"))),
        "kda_prologue": dict(ms=round(pro_ms, 4), **roofline(
            "hbm", PROLOGUE_BYTES_PER_TH * th, pro_ms, hbm, "GB/s", recorded_traffic("kda_prologue"))),
        "kda_chunk_fwd": dict(ms=round(chk_ms, 4), launches=2, **roofline(
            "hbm", CHUNK_BYTES_PER_TH * th, chk_ms, hbm, "GB/s", recorded_traffic("kda_chunk_fwd"))),
        "kda_chunk_fwd_gated": dict(ms=round(gated_ms, 4), launches=2, **roofline(
            "hbm", GATED_BYTES_PER_TH * th, gated_ms, hbm, "GB/s",
            recorded_traffic("kda_chunk_fwd_gated"))),
        "kda_output_epilogue": dict(ms=round(epi_ms, 4), **roofline(
            "hbm", EPILOGUE_BYTES_PER_TH * th, epi_ms, hbm, "GB/s",
            recorded_traffic("kda_output_epilogue"))),
        "kda_chunk_bwd": dict(ms=round(bwd_ms, 4), launches=4, **roofline(
            "hbm", BWD_BYTES_PER_TH * th, bwd_ms, hbm, "GB/s", recorded_traffic("kda_chunk_bwd"))),
        "kda_chunk_fwd_windowed64": dict(
            ms=round(windowed_ms, 4), window_chunks=win_chunks,
            launches=2 * (((T + 63) // 64 + 1 + win_chunks - 1) // win_chunks),
            workspace_gb=round(win_ws_gb, 3), full_workspace_gb=round(ws.numel() / 1e9, 3),
            **roofline("hbm", CHUNK_BYTES_PER_TH_PLAN * th, windowed_ms, hbm, "GB/s",
                       recorded_traffic("kda_chunk_fwd_windowed64"))),
        "kda_chunk_fwd_one_pass": dict(ms=round(one_pass_ms, 4), **roofline(
            "hbm", CHUNK_BYTES_PER_TH * th, one_pass_ms, hbm, "GB/s",
            recorded_traffic("kda_chunk_fwd_one_pass"))),
    }
    kernels["kda_chunk_fwd"]["tensor_tflops"] = round(
        CHUNK_FLOPS_PER_TH * th / (chk_ms * 1e-3) / 1e12, 2)
    dominant = "kda_chunk_fwd"
    roof = roofline("hbm", CHUNK_BYTES_PER_TH_PLAN * th, chk_ms, hbm, "GB/s",
                    recorded_traffic("kda_chunk_fwd"))
    roof["kernel"] = dominant + " (one call: prep pass + state pass)"
    roof["peak_source"] = f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
    roof["algorithmic_bytes_per_token_head"] = CHUNK_BYTES_PER_TH_PLAN
    roof["frac_fp32_readout_bytes"] = kernels[dominant]["frac"]  # 1796 B: o written as fp32
    # the whole step against the HBM floor of the fused workload (x in, g, beta, o out)
    fused_floor_ms = 1e3 * (3 * D_ * 2 + D_ * 4 + 4 + D_ * 2) * th / (hbm * 1e9)

    # ---- end to end through the C ABI with host buffers ----
    # Every step copies its inputs in from pinned host memory and its read-out back.
    # Three streams with double-buffered inputs and outputs: step i+1's inputs
    # travel host -> device while step i computes and its read-out travels
    # device -> host (the two directions of the host link run at the same time).
    e2e_steps = max(2, args.e2e_steps)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    xs, gs, bs = [x, torch.empty_like(x)], [g, torch.empty_like(g)], [beta, torch.empty_like(beta)]
    outs = [o, torch.empty_like(o)]
    out_host = [torch.empty((T, H, D), dtype=torch.float32, pin_memory=True) for _ in range(2)]
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(s_in)
    for i in range(e2e_steps):
        b = i % 2
        if i >= 2:
            s_in.wait_event(comp_done[b])   # step i-2 has read slot b
        with torch.cuda.stream(s_in):
            xs[b].copy_(inp.x, non_blocking=True)
            gs[b].copy_(inp.g, non_blocking=True)
            bs[b].copy_(inp.beta, non_blocking=True)
        in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        if i >= 2:
            stream.wait_event(out_done[b])  # step i-2's read-out has left slot b
        kda.kda_prologue(xs[b], w, q, k, v, H=H, D=D, stream=stream)
        kda.kda_chunk_fwd(q, k, v, gs[b], bs[b], outs[b], scale=inp.scale, final_state=fs,
                          chunk=inp.chunk, workspace=ws, stream=stream)
        comp_done[b].record(stream)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            out_host[b].copy_(outs[b], non_blocking=True)
        out_done[b].record(s_out)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    assert kda.kda_get_device_status() == 0
    e2e_value, e2e_ms = job_throughput(world, T, e0.elapsed_time(e1) / e2e_steps)
    h2d = inp.x.numel() * 2 + inp.g.numel() * 4 + inp.beta.numel() * 4
    d2h = out_host[0].numel() * 4
    del x, o, g, beta, inp, ws, xs, gs, bs, outs, out_host
    torch.cuda.empty_cache()

    # ---- batched decode: 256 sequences x 96 heads, consecutive steps ----
    dinp = W.decode256(steps=args.decode_steps)
    Nd, Hd, Dd = dinp.N, dinp.H, dinp.D
    state = dinp.state.to(dev)
    cache = dinp.conv_cache.to(dev)
    dw = dinp.conv_w.to(dev)
    dx, dg, db = dinp.x.to(dev), dinp.g.to(dev), dinp.beta.to(dev)
    do = torch.empty((Nd, Hd, Dd), dtype=torch.float32, device=dev)
    wstate, wcache = state.clone(), cache.clone()  # warm-up on copies: the timed steps
    for s in range(min(3, args.decode_steps)):    # start from the workload's state
        kda.kda_decode_step(dx[s], dw, wcache, dg[s], db[s], wstate, do, H=Hd, D=Dd,
                            scale=dinp.scale, stream=stream)
    torch.cuda.synchronize(dev)
    del wstate, wcache
    dev_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
              for _ in range(args.decode_steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for s in range(args.decode_steps):
        dev_ev[s][0].record(stream)
        kda.kda_decode_step(dx[s], dw, cache, dg[s], db[s], state, do, H=Hd, D=Dd,
                            scale=dinp.scale, stream=stream)
        dev_ev[s][1].record(stream)
    d1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier(world)
    assert kda.kda_get_device_status() == 0
    dec_value, dec_ms = job_throughput(world, Nd, d0.elapsed_time(d1) / args.decode_steps)
    dec_kernel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in dev_ev)
    decode = {
        "metric": "decode tokens/s", "unit": "tokens/s",
        "value": round(dec_value, 1),
        "ms_per_step": round(dec_ms, 4), "steps": args.decode_steps,
        "workload": "decode256: 256 sequences x 96 heads x d=128, fp32 state in place, "
                    "bf16 projections with conv cache",
        "roofline": dict(roofline("hbm", DECODE_BYTES_PER_SH * Nd * Hd, dec_kernel_ms, hbm,
                                  "GB/s", recorded_traffic("kda_decode_step")),
                         kernel="kda_decode_step"),
    }
    launches_total = launches
    if rank == 0:  # the oracle's run of the same 100 steps on 16 of the 256 sequences
        decode["parity"] = decode_parity(state, cache, do, args.decode_steps,
                                         list(range(0, Nd, Nd // 16)))
    del state, cache, dx, dg, db

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": k3_config(world, T, H, D),
        "roofline": roof,
        "kernels": kernels,
        "fused_hbm_floor_ms": round(fused_floor_ms, 4),
        "step_fraction_of_fused_floor": round(fused_floor_ms / ms_step, 4),
        "decode": decode,
        "seq4k": seq4k,
        "varlen16": varlen,
        "tiny_f32": tiny,
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "pipeline": "three streams, inputs and outputs double-buffered: step i+1's "
                            "inputs are copied in while step i computes and its o is "
                            "copied out"},
        "gpu_launches": launches_total,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_tokens)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_ncu_case(args):
    """Launch one kernel twice (warm-up, then the launch to capture) on a slice
    of the workload, for profiling runs; prints nothing."""
    import gated_delta_rule_prologue_b200 as kda
    dev = torch.device("cuda", 0)
    if args.ncu_case in ("seq4k", "seq4k_whole"):
        sinp = W.seq4k_bf16()
        args4 = [t.to(dev) for t in (sinp.q, sinp.k, sinp.v, sinp.g, sinp.beta)]
        s04 = sinp.initial_state.to(dev)
        o = torch.empty(sinp.q.shape, device=dev)
        fs = torch.empty_like(s04)
        seg = None if args.ncu_case == "seq4k" else 0
        for _ in range(2):
            kda.kda_chunk_fwd(*args4, o, scale=sinp.scale, initial_state=s04, final_state=fs,
                              segment_chunks=seg)
    elif args.ncu_case == "decode":
        d = W.decode256(steps=2)
        state, cache = d.state.to(dev), d.conv_cache.to(dev)
        w = d.conv_w.to(dev)
        o = torch.empty((d.N, d.H, d.D), device=dev)
        for s_ in range(2):
            kda.kda_decode_step(d.x[s_].to(dev), w, cache, d.g[s_].to(dev), d.beta[s_].to(dev),
                                state, o, H=d.H, D=d.D)
    else:
        inp = W.k3_prefill()
        T = min(args.ncu_tokens, inp.T)
        H, D = inp.H, inp.D
        x = inp.x[:T].contiguous().to(dev)
        w = inp.conv_w.to(dev)
        g = inp.g[:T].contiguous().to(dev)
        beta = inp.beta[:T].contiguous().to(dev)
        o = torch.empty((T, H, D), device=dev)
        q = torch.empty((T, H, D), dtype=torch.float16, device=dev)
        k, v = torch.empty_like(q), torch.empty_like(q)
        for _ in range(2):
            if args.ncu_case == "fused":
                kda.kda_prologue_chunk_fwd(x, w, g, beta, o, H=H, D=D)
            elif args.ncu_case == "prologue":
                kda.kda_prologue(x, w, q, k, v, H=H, D=D)
            elif args.ncu_case == "bwd":
                kda.kda_prologue(x, w, q, k, v, H=H, D=D)
                d_o = torch.randn((T, H, D), generator=torch.Generator().manual_seed(3)).to(dev)
                kda.kda_chunk_bwd(q, k, v, g, beta, d_o, want_d_initial_state=False)
            elif args.ncu_case == "chunk_one_pass":
                kda.kda_prologue(x, w, q, k, v, H=H, D=D)
                kda.kda_chunk_fwd(q, k, v, g, beta, o, workspace=None)
            else:
                kda.kda_prologue(x, w, q, k, v, H=H, D=D)
                kda.kda_chunk_fwd(q, k, v, g, beta, o)
    torch.cuda.synchronize(dev)
    assert kda.kda_get_device_status() == 0


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--decode-steps", type=int, default=100)
    ap.add_argument("--e2e-steps", type=int, default=4)
    ap.add_argument("--cpu-tokens", type=int, default=ORACLE_SAMPLE_TOKENS)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ncu-case", choices=("fused", "prologue", "chunk", "chunk_one_pass", "decode",
                                           "seq4k", "seq4k_whole", "bwd"),
                    help="profiling mode: launch one kernel twice on a workload slice and exit")
    ap.add_argument("--ncu-tokens", type=int, default=4096)
    args = ap.parse_args()
    if args.ncu_case:
        run_ncu_case(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_setup(args) if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if args.impl == "ours" and world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
