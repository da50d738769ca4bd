"""GPU parity on the recurrence's degenerate gates and on the decode step's
smaller head sizes and input types, against the float64 oracle.

- beta = 0 with no decay (g = 0): the delta write vanishes and the state is
  carried unchanged, S_t = S_0, so o_t = scale * S_0^T q_t.  Every path keeps
  S_0 to fp32 rounding (the tensor-core path's update is S + K'^T U with U = 0
  exactly, the decode step's s' + 0 * e * k).
- beta = 1: each token's key slot is overwritten with its value (the delta
  rule's full projection step); no closed form, checked against the oracle.
- Decode at D in {16, 32, 64, 128} with bf16, fp16 and fp32 projections:
  the kernel's warp layouts differ per D (lanes per row, rows per warp).
Tolerances: fp32 arithmetic paths 1e-4 of the RMS, bf16/fp16-operand paths
2e-2 of the RMS and 1e-2 relative Frobenius for the state.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import kda_decode_step as o_decode, kda_recurrent, state_from_abi, state_to_abi

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_F32, TOL_BF16, TOL_STATE = 1e-4, 2e-2, 1e-2
PASSES = {"two_pass": "auto", "one_pass": None}


@pytest.fixture(scope="module")
def kda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import gated_delta_rule_prologue_b200 as m
    return m


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_max(got, ref):
    assert np.all(np.isfinite(got))
    return float(np.max(np.abs(got - ref)) / np.sqrt(np.mean(ref * ref)))


def rel_fro(got, ref):
    assert np.all(np.isfinite(got))
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def run_prefill(kda, inp, workspace):
    q, k, v = inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(DEV)
    N, H, D = inp.N, inp.H, inp.q.shape[2]
    o = torch.empty((inp.T, H, D), dtype=torch.float32, device=DEV)
    fs = torch.empty((N, H, D, D), device=DEV)
    kda.kda_chunk_fwd(q, k, v, inp.g.to(DEV), inp.beta.to(DEV), o, scale=inp.scale,
                      initial_state=inp.initial_state.to(DEV), final_state=fs, cu_seqlens=cu,
                      chunk=inp.chunk, workspace=workspace)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    return f64(o), f64(fs)


def oracle_prefill(inp):
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy()
    o, S = kda_recurrent(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.scale,
                         state_from_abi(inp.initial_state), cu)
    return o, state_to_abi(S)


@pytest.mark.parametrize("passes", list(PASSES))
@pytest.mark.parametrize("bf16", [True, False], ids=["tensor_core", "cuda_core_f32"])
def test_prefill_beta_zero_no_decay_carries_the_state(kda, bf16, passes):
    if passes == "one_pass" and not bf16:
        pytest.skip("only the tensor-core path has two variants")
    inp = W.random_prefill(300, 200, 2, 128, bf16=bf16, s0_std=0.2, lengths=[130, 70],
                           g_fn=lambda z: torch.zeros_like(z))
    inp.beta = torch.zeros_like(inp.beta)
    inp.scale = 0.5
    o, S = run_prefill(kda, inp, PASSES[passes])
    o_ref, S_ref = oracle_prefill(inp)
    s0 = f64(inp.initial_state)
    np.testing.assert_allclose(S_ref, s0, rtol=0, atol=0)  # the oracle's closed form
    assert rel_fro(S, s0) <= 1e-6
    assert rel_max(o, o_ref) <= (TOL_BF16 if bf16 else TOL_F32)


@pytest.mark.parametrize("passes", list(PASSES))
def test_prefill_beta_one(kda, passes):
    """Full overwrite on every token, moderate decay, two packed sequences with a
    ragged last chunk each."""
    inp = W.random_prefill(301, 250, 2, 128, s0_std=0.1, lengths=[150, 100],
                           g_fn=lambda z: -5.0 * torch.sigmoid(z - 3.0))
    inp.beta = torch.ones_like(inp.beta)
    o, S = run_prefill(kda, inp, PASSES[passes])
    o_ref, S_ref = oracle_prefill(inp)
    assert rel_max(o, o_ref) <= TOL_BF16
    assert rel_fro(S, S_ref) <= TOL_STATE


def decode_problem(D, dtype, steps, N=5, H=3, seed=0):
    C = 3 * H * D
    r = torch.Generator().manual_seed(700 + D + seed)
    x = torch.randn((steps, N, C), generator=r).to(dtype)
    w = 0.5 * torch.randn((C, 4), generator=r)
    cache = torch.randn((N, 3, C), generator=r).to(dtype)
    g = -5.0 * torch.sigmoid(torch.randn((steps, N, H, D), generator=r) - 2.0)
    beta = torch.sigmoid(torch.randn((steps, N, H), generator=r))
    s0 = 0.1 * torch.randn((N, H, D, D), generator=r)
    return x, w, cache, g, beta, s0


def run_decode(kda, x, w, cache, g, beta, s0, H, D, scale):
    state, cache_d = s0.to(DEV).clone(), cache.to(DEV).clone()
    outs = []
    for s in range(x.shape[0]):
        o = torch.empty((x.shape[1], H, D), dtype=torch.float32, device=DEV)
        kda.kda_decode_step(x[s].to(DEV), w.to(DEV), cache_d, g[s].to(DEV), beta[s].to(DEV),
                            state, o, H=H, D=D, scale=scale)
        outs.append(o)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    return [f64(o) for o in outs], f64(state), f64(cache_d)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32],
                         ids=["bf16", "f16", "f32"])
@pytest.mark.parametrize("D", [16, 32, 64, 128])
def test_decode_head_sizes_and_input_types(kda, D, dtype):
    """Four consecutive steps of five sequences x three heads; the decode step
    computes in fp32 from the given projections, so it meets the fp32 bound."""
    H, steps = 3, 4
    x, w, cache, g, beta, s0 = decode_problem(D, dtype, steps, H=H)
    outs, state, cache_out = run_decode(kda, x, w, cache, g, beta, s0, H, D, 0.5)
    S, c = state_from_abi(s0), cache
    for s in range(steps):
        o_ref, S, c = o_decode(x[s], w, c, g[s], beta[s], S, H, D, scale=0.5)
        assert rel_max(outs[s], o_ref) <= TOL_F32, s
    assert rel_fro(state, state_to_abi(S)) <= 1e-5
    np.testing.assert_array_equal(cache_out, np.asarray(c, dtype=np.float64))


@pytest.mark.parametrize("D", [16, 128])
def test_decode_beta_zero_no_decay_keeps_the_state(kda, D):
    """beta = 0, g = 0: s' = S and the write adds 0 * e * k, so the state comes
    back bit-identical and o = scale * S^T q."""
    H, steps = 3, 2
    x, w, cache, g, beta, s0 = decode_problem(D, torch.bfloat16, steps, H=H, seed=1)
    g, beta = torch.zeros_like(g), torch.zeros_like(beta)
    outs, state, _ = run_decode(kda, x, w, cache, g, beta, s0, H, D, 1.0)
    np.testing.assert_array_equal(state, f64(s0))
    S, c = state_from_abi(s0), cache
    for s in range(steps):
        o_ref, S, c = o_decode(x[s], w, c, g[s], beta[s], S, H, D)
        assert rel_max(outs[s], o_ref) <= TOL_F32
