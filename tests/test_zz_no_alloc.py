"""kda_chunk_fwd_static (scratch in the library's fixed device buffer, no
allocation) against kda_chunk_fwd_ws (caller-owned workspace) on the same
inputs, two calls in a row: both run the same kernels, so the results must
be bit-identical, call after call.  The file name sorts last so that the
test also runs after every other GPU test; it depends on nothing they leave
behind and passes alone."""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_caller_workspace_two_calls_in_a_row():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import gated_delta_rule_prologue_b200 as kda
    kda.kda_get_device_status()  # start from a clear status word
    inp = W.seq4k_bf16()         # T=4096, H=8, d=128, chunk 64: the two-pass path
    dev = "cuda"
    N, T, H, D = inp.N, inp.T, inp.H, inp.q.shape[2]
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    g, beta = inp.g.to(dev), inp.beta.to(dev)
    s0 = inp.initial_state.to(dev).contiguous()
    need = kda.kda_chunk_fwd_workspace_bytes(N, T, H, D, D, 64, q.dtype)
    assert 0 < need <= kda.KDA_CHUNK_STATIC_SCRATCH_BYTES
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    for _ in range(2):
        o_ws = torch.empty((T, H, D), device=dev)
        s_ws = torch.empty((N, H, D, D), device=dev)
        kda.kda_chunk_fwd(q, k, v, g, beta, o_ws, scale=inp.scale, initial_state=s0,
                          final_state=s_ws, workspace=ws)
        o_st = torch.full((T, H, D), float("nan"), device=dev)
        s_st = torch.full((N, H, D, D), float("nan"), device=dev)
        kda.kda_chunk_fwd_static(q, k, v, g, beta, o_st, scale=inp.scale, initial_state=s0,
                                 final_state=s_st)
        torch.cuda.synchronize()
        assert kda.kda_get_device_status() == 0
        np.testing.assert_array_equal(o_st.cpu().numpy(), o_ws.cpu().numpy())
        np.testing.assert_array_equal(s_st.cpu().numpy(), s_ws.cpu().numpy())
        assert np.all(np.isfinite(o_st.cpu().numpy()))
