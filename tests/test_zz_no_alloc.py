"""kda_chunk_fwd_static: the two-pass prefill for callers that cannot
allocate device memory (code running under a memory pool or allocator they do
not own, inside a region where cudaMalloc would synchronise the device, or a
runtime that has handed all memory out up front).  Its scratch is the
library's fixed __device__ array, and its status word is a __device__ int, so
the call allocates nothing.

Each case compares it with kda_chunk_fwd_ws (caller-owned workspace) on the
same inputs, two calls in a row.  Both run the same kernels, so the results
must be bit-identical, call after call.  One case runs in a fresh process in
which kda_chunk_fwd_static is the first library call on the device, and
checks the device's free memory: the first call may only load the library's
device modules (the 64 MiB array and kernel code), and later calls must not
change it at all.  The file name sorts last so that a run that stops at the
first failure has run every other test; the cases depend on nothing the other
tests leave behind and pass alone."""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _both_paths_twice(inp, dev="cuda"):
    import gated_delta_rule_prologue_b200 as kda
    N, T, H, D = inp.N, inp.T, inp.H, inp.q.shape[2]
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    g, beta = inp.g.to(dev), inp.beta.to(dev)
    s0 = None if inp.initial_state is None else inp.initial_state.to(dev).contiguous()
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(dev)
    need = kda.kda_chunk_fwd_workspace_bytes(N, T, H, D, D, 64, q.dtype)
    assert 0 < need <= kda.KDA_CHUNK_STATIC_SCRATCH_BYTES
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    for _ in range(2):
        o_ws = torch.empty((T, H, D), device=dev)
        s_ws = torch.empty((N, H, D, D), device=dev)
        kda.kda_chunk_fwd(q, k, v, g, beta, o_ws, scale=inp.scale, initial_state=s0,
                          final_state=s_ws, cu_seqlens=cu, workspace=ws)
        o_st = torch.full((T, H, D), float("nan"), device=dev)
        s_st = torch.full((N, H, D, D), float("nan"), device=dev)
        kda.kda_chunk_fwd_static(q, k, v, g, beta, o_st, scale=inp.scale, initial_state=s0,
                                 final_state=s_st, cu_seqlens=cu)
        torch.cuda.synchronize()
        assert kda.kda_get_device_status() == 0
        np.testing.assert_array_equal(o_st.cpu().numpy(), o_ws.cpu().numpy())
        np.testing.assert_array_equal(s_st.cpu().numpy(), s_ws.cpu().numpy())
        assert np.all(np.isfinite(o_st.cpu().numpy()))


def test_static_scratch_matches_caller_workspace_two_calls_in_a_row():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import gated_delta_rule_prologue_b200 as kda
    kda.kda_get_device_status()  # start from a clear status word
    _both_paths_twice(W.seq4k_bf16())  # T=4096, H=8: the split (segmented) state pass


def test_static_scratch_varlen_matches_caller_workspace():
    """Packed sequences: the index pass writes the chunk index into the shared
    array on every call (ragged lengths, one shorter than a chunk, one empty)."""
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    lengths = [700, 64, 1, 0, 1300, 129]
    inp = W.random_prefill(61, sum(lengths), 4, 128, lengths=lengths, s0_std=0.02)
    _both_paths_twice(inp)


_FRESH = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r})
    import numpy as np
    import torch
    import workloads as W
    import gated_delta_rule_prologue_b200 as kda

    torch.cuda.init()
    inp = W.seq4k_bf16()
    dev = "cuda"
    N, T, H, D = inp.N, inp.T, inp.H, inp.q.shape[2]
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    g, beta = inp.g.to(dev), inp.beta.to(dev)
    s0 = inp.initial_state.to(dev).contiguous()
    outs = [(torch.empty((T, H, D), device=dev), torch.empty((N, H, D, D), device=dev))
            for _ in range(3)]
    torch.cuda.synchronize()
    free = [torch.cuda.mem_get_info()[0]]
    for o, s in outs:  # the first library call on this device is kda_chunk_fwd_static
        kda.kda_chunk_fwd_static(q, k, v, g, beta, o, scale=inp.scale, initial_state=s0,
                                 final_state=s)
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
    assert kda.kda_get_device_status() == 0
    ws = torch.empty(kda.kda_chunk_fwd_workspace_bytes(N, T, H, D, D, 64, q.dtype),
                     dtype=torch.uint8, device=dev)
    o_ws = torch.empty((T, H, D), device=dev)
    s_ws = torch.empty((N, H, D, D), device=dev)
    kda.kda_chunk_fwd(q, k, v, g, beta, o_ws, scale=inp.scale, initial_state=s0,
                      final_state=s_ws, workspace=ws)
    torch.cuda.synchronize()
    for o, s in outs:
        np.testing.assert_array_equal(o.cpu().numpy(), o_ws.cpu().numpy())
        np.testing.assert_array_equal(s.cpu().numpy(), s_ws.cpu().numpy())
    print("FREE", *free)
""")


def test_static_scratch_first_call_in_fresh_process_allocates_nothing():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    env = dict(os.environ, CUDA_MODULE_LOADING="LAZY")
    r = subprocess.run([sys.executable, "-c", _FRESH.format(root=ROOT)], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("FREE")][-1]
    free = [int(t) for t in line.split()[1:]]
    first = free[0] - free[1]
    # the first call loads device modules: the 64 MiB array plus kernel code
    assert 0 <= first <= (64 << 20) + (64 << 20), first
    # later calls leave the device's free memory exactly as it was
    assert free[2] == free[1] and free[3] == free[1], free
