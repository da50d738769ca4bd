"""Failure detection on the GPU without a fault: a bounded device wait is made
to run out (an mbarrier that nothing arrives at, 1 ms limit).  The kernel
records KDA_ERR_DEVICE_TIMEOUT in the status word and returns, so the context
stays usable: a prefill right after it on the same context is correct and
leaves the status word clear."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import kda_recurrent, state_from_abi, state_to_abi

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import gated_delta_rule_prologue_b200 as kda
    kda.kda_get_device_status()  # clear
    kda.kda_selftest_wait_timeout(1000)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == kda.KDA_ERR_DEVICE_TIMEOUT
    assert kda.kda_get_device_status() == 0  # reading clears it

    inp = W.random_prefill(77, 300, 2, 128, s0_std=0.02)
    dev = "cuda"
    o = torch.empty(inp.v.shape, dtype=torch.float32, device=dev)
    fs = torch.empty((1, 2, 128, 128), device=dev)
    kda.kda_chunk_fwd(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.g.to(dev),
                      inp.beta.to(dev), o, initial_state=inp.initial_state.to(dev),
                      final_state=fs, workspace="auto")
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    f = lambda t: t.double().numpy()
    o_ref, s_ref = kda_recurrent(f(inp.q), f(inp.k), f(inp.v), f(inp.g), f(inp.beta),
                                 initial_state=state_from_abi(f(inp.initial_state)))
    got = o.cpu().double().numpy()
    assert np.max(np.abs(got - o_ref)) / np.sqrt(np.mean(o_ref ** 2)) <= 2e-2
    s_got = fs.cpu().double().numpy()
    s_ref = state_to_abi(s_ref)
    assert np.linalg.norm(s_got - s_ref) / np.linalg.norm(s_ref) <= 1e-2
