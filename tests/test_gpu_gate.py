"""GPU parity of the in-kernel bounded gate ([W1 彩蛋], the gate.py excerpt):
the *_gated entry points take gate pre-activations g_raw and compute
g = lower_bound * sigmoid(exp(A_log[h]) * (g_raw + dt_bias[h, :])) in the
kernels.  Compared with the oracle (gate, then the recurrence) at the bf16
tolerances, and with the ungated path fed the oracle's gate."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import gate, kda_decode_step as o_decode, kda_recurrent, prologue as o_prologue
from oracle import state_from_abi, state_to_abi

pytestmark = pytest.mark.gpu

TOL_BF16, TOL_STATE = 2e-2, 1e-2
DEV = "cuda"


@pytest.fixture(scope="module")
def kda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import gated_delta_rule_prologue_b200 as m
    return m


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_max(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got))
    return float(np.max(np.abs(got - ref)) / np.sqrt(np.mean(ref * ref)))


def rel_fro(got, ref):
    return float(np.linalg.norm(np.asarray(got) - ref) / np.linalg.norm(ref))


def gate_params(seed, T, H, D, dtype=torch.bfloat16):
    r = torch.Generator().manual_seed(seed)
    g_raw = torch.randn((T, H, D), generator=r).to(dtype)
    A_log = 0.5 * torch.randn((H,), generator=r)
    dt_bias = torch.randn((H, D), generator=r)
    return g_raw, A_log, dt_bias


@pytest.mark.parametrize("params", ["both", "none"])
def test_chunk_gated_matches_oracle(kda, params):
    lengths = [130, 0, 64, 257]
    inp = W.random_prefill(40, sum(lengths), 3, 128, s0_std=0.05, lengths=lengths)
    T, H, D, N = inp.T, inp.H, 128, inp.N
    g_raw, A_log, dt_bias = gate_params(41, T, H, D)
    if params == "none":
        A_log = dt_bias = None
    g = gate(g_raw, None if A_log is None else A_log.numpy(),
             None if dt_bias is None else dt_bias.numpy(), -5.0)
    o = torch.empty((T, H, D), device=DEV)
    fs = torch.empty((N, H, D, D), device=DEV)
    kda.kda_chunk_fwd_gated(inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV), g_raw.to(DEV),
                            inp.beta.to(DEV), o, A_log=None if A_log is None else A_log.to(DEV),
                            dt_bias=None if dt_bias is None else dt_bias.to(DEV),
                            initial_state=inp.initial_state.to(DEV), final_state=fs,
                            cu_seqlens=inp.cu_seqlens.to(DEV))
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    o_ref, S_ref = kda_recurrent(inp.q, inp.k, inp.v, g, inp.beta, 1.0,
                                 state_from_abi(inp.initial_state), inp.cu_seqlens.numpy())
    assert rel_max(f64(o), o_ref) <= TOL_BF16
    assert rel_fro(f64(fs), state_to_abi(S_ref)) <= TOL_STATE


def test_gated_equals_ungated_fed_the_same_gate(kda):
    """The kernel's fp32 gate against the oracle's gate passed as fp32 g: the
    two calls differ only by the gate's rounding."""
    inp = W.random_prefill(42, 300, 2, 128, s0_std=0.05, lengths=[300])
    T, H, D = inp.T, inp.H, 128
    g_raw, A_log, dt_bias = gate_params(43, T, H, D)
    g = torch.from_numpy(gate(g_raw, A_log.numpy(), dt_bias.numpy(), -5.0)).float()
    q, k, v, b = inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV), inp.beta.to(DEV)
    o1 = torch.empty((T, H, D), device=DEV)
    o2 = torch.empty_like(o1)
    kda.kda_chunk_fwd_gated(q, k, v, g_raw.to(DEV), b, o1, A_log=A_log.to(DEV),
                            dt_bias=dt_bias.to(DEV))
    kda.kda_chunk_fwd(q, k, v, g.to(DEV), b, o2)
    torch.cuda.synchronize()
    assert rel_max(f64(o1), f64(o2)) <= 2e-3


def test_fused_gated_matches_oracle_with_cache(kda):
    H, D = 2, 128
    lengths = [70, 0, 200, 3]
    T, N, C = sum(lengths), len(lengths), 3 * H * D
    r = torch.Generator().manual_seed(44)
    x = torch.randn((T, C), generator=r).to(torch.bfloat16)
    w = 0.5 * torch.randn((C, 4), generator=r)
    beta = torch.sigmoid(torch.randn((T, H), generator=r))
    cache0 = torch.randn((N, 3, C), generator=r).to(torch.bfloat16)
    s0 = 0.05 * torch.randn((N, H, D, D), generator=r)
    g_raw, A_log, dt_bias = gate_params(45, T, H, D)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    o = torch.empty((T, H, D), device=DEV)
    fs = torch.empty((N, H, D, D), device=DEV)
    cache_out = torch.empty((N, 3, C), dtype=torch.bfloat16, device=DEV)
    kda.kda_prologue_chunk_fwd_gated(x.to(DEV), w.to(DEV), g_raw.to(DEV), beta.to(DEV), o, H=H,
                                     D=D, A_log=A_log.to(DEV), dt_bias=dt_bias.to(DEV),
                                     cache_in=cache0.to(DEV), cache_out=cache_out,
                                     initial_state=s0.to(DEV), final_state=fs,
                                     cu_seqlens=torch.tensor(cu, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    qr, kr, vr, c_ref = o_prologue(x, w, H, D, cu, cache0)
    g = gate(g_raw, A_log.numpy(), dt_bias.numpy(), -5.0)
    o_ref, S_ref = kda_recurrent(qr, kr, vr, g, beta, 1.0, state_from_abi(s0), cu)
    assert rel_max(f64(o), o_ref) <= TOL_BF16
    assert rel_fro(f64(fs), state_to_abi(S_ref)) <= TOL_STATE
    np.testing.assert_array_equal(f64(cache_out), c_ref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_gated_matches_oracle(kda, dtype):
    N, H, D = 5, 3, 128
    C = 3 * H * D
    r = torch.Generator().manual_seed(46)
    x = torch.randn((N, C), generator=r).to(dtype)
    w = 0.5 * torch.randn((C, 4), generator=r)
    cache = torch.randn((N, 3, C), generator=r).to(dtype)
    beta = torch.sigmoid(torch.randn((N, H), generator=r))
    state = 0.05 * torch.randn((N, H, D, D), generator=r)
    g_raw, A_log, dt_bias = gate_params(47, N, H, D, dtype)
    o = torch.empty((N, H, D), device=DEV)
    st = state.to(DEV).contiguous()
    cache_d = cache.to(DEV).contiguous()
    kda.kda_decode_step_gated(x.to(DEV), w.to(DEV), cache_d, g_raw.to(DEV), beta.to(DEV), st, o,
                              H=H, D=D, A_log=A_log.to(DEV), dt_bias=dt_bias.to(DEV),
                              lower_bound=-4.0)
    torch.cuda.synchronize()
    g = gate(g_raw, A_log.numpy(), dt_bias.numpy(), -4.0)
    o_ref, S_ref, c_ref = o_decode(x, w, cache, g, beta, state_from_abi(state), H, D)
    tol = 1e-4 if dtype == torch.float32 else TOL_BF16
    assert rel_max(f64(o), o_ref) <= tol
    assert rel_fro(f64(st), state_to_abi(S_ref)) <= (1e-5 if dtype == torch.float32 else TOL_STATE)
