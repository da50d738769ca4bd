"""GPU parity of the output epilogue ([W1 第六站]: per-head RMSNorm of the
read-out, then the sigmoid output gate) against the float64 oracle: each output
within the rounding of its storage type plus fp32 noise; and the whole
prefill-then-epilogue path against the oracle recurrence followed by the
oracle epilogue."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import kda_recurrent, output_epilogue

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROUNDOFF = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11, torch.float32: 0.0}


@pytest.fixture(scope="module")
def kda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import gated_delta_rule_prologue_b200 as m
    return m


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("D", [128, 64, 16])
def test_epilogue_matches_oracle(kda, dtype, D):
    T, H = 301, 3
    r = torch.Generator().manual_seed(60 + D)
    o = 3.0 * torch.randn((T, H, D), generator=r)
    o[7, 1] = 0.0                                  # an all-zero row: eps keeps it finite
    gate = (2.0 * torch.randn((T, H, D), generator=r)).to(dtype)
    weight = 0.5 + torch.rand((D,), generator=r)
    out = torch.empty((T, H, D), dtype=dtype, device=DEV)
    kda.kda_output_epilogue(o.to(DEV), gate.to(DEV), weight.to(DEV), out, eps=1e-5)
    torch.cuda.synchronize()
    ref = output_epilogue(o, gate, weight, 1e-5)
    got = f64(out)
    rms = np.sqrt(np.mean(ref * ref))
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - ref) <= ROUNDOFF[dtype] * np.abs(ref) + 2e-6 * np.abs(ref) + 1e-6 * rms)
    assert np.all(got[7, 1] == 0.0)


def test_prefill_then_epilogue(kda):
    """The epilogue applied to kda_chunk_fwd's read-out equals the oracle
    epilogue of that same read-out (storage rounding, elementwise), and the
    read-out's error carried through the epilogue stays within the bf16 bound
    of the oracle recurrence + oracle epilogue on rows whose read-out RMS is at
    least half the global one (RMSNorm divides a row by its own RMS, so the
    read-out's absolute error grows by RMS_global / RMS_row on small rows)."""
    inp = W.seq4k_bf16()
    T, H, D = inp.T, inp.H, 128
    o = torch.empty((T, H, D), device=DEV)
    kda.kda_chunk_fwd(inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV), inp.g.to(DEV),
                      inp.beta.to(DEV), o, initial_state=inp.initial_state.to(DEV))
    r = torch.Generator().manual_seed(65)
    gate = torch.randn((T, H, D), generator=r).to(torch.bfloat16)
    weight = 0.5 + torch.rand((D,), generator=r)
    out = torch.empty((T, H, D), dtype=torch.bfloat16, device=DEV)
    kda.kda_output_epilogue(o, gate.to(DEV), weight.to(DEV), out)
    torch.cuda.synchronize()
    got = f64(out)
    mine = output_epilogue(f64(o), gate, weight, 1e-5)
    assert np.all(np.abs(got - mine) <= (2.0 ** -8 + 2e-6) * np.abs(mine)
                  + 1e-6 * np.sqrt(np.mean(mine * mine)))
    from oracle import state_from_abi
    o_ref, _ = kda_recurrent(inp.q, inp.k, inp.v, inp.g, inp.beta, 1.0,
                             state_from_abi(inp.initial_state))
    ref = output_epilogue(o_ref, gate, weight, 1e-5)
    row_rms = np.sqrt(np.mean(o_ref * o_ref, axis=-1))
    keep = row_rms >= 0.5 * np.sqrt(np.mean(o_ref * o_ref))
    assert keep.mean() > 0.5
    # the read-out's error carried through the epilogue (the output's own bf16
    # rounding, up to 2^-9 of values near 10x the RMS, is checked above)
    err = np.max(np.abs(mine - ref)[keep]) / np.sqrt(np.mean(ref[keep] ** 2))
    assert err <= 2e-2
