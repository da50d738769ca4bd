"""GPU parity of the sequence-parallel state pass.

The chunk update is an affine map of the entry state ("KimiK3轻量化复刻实现KDA
并行解析，Chunkwise并行与状态压缩机制详解", Figure 1 and Figure 3), so the
state pass can cut each sequence into segments: a transition pass computes
every segment's map, an fp32 scan composes the entry states, and the output
pass runs all segments at once.  kda_chunk_fwd_segmented_ws takes the segment
length explicitly, so short inputs here reach many segments per sequence,
ragged segment lengths, one-chunk segments and unsplit sequences in one
batch.  Compared with the float64 oracle at the bf16 tolerances, with the
unsplit state pass, and for bit-identical reruns.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import gate, kda_recurrent, state_from_abi, state_to_abi

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
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got))
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def run_seg(kda, inp, L, *, in_place=False, workspace="auto"):
    q, k, v = inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV)
    g, beta = inp.g.to(DEV), inp.beta.to(DEV)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(DEV)
    N, H, D = inp.N, inp.H, inp.q.shape[2]
    s0 = None if inp.initial_state is None else inp.initial_state.to(DEV).contiguous()
    fs = s0 if (in_place and s0 is not None) else torch.empty((N, H, D, D), device=DEV)
    o = torch.empty(v.shape, dtype=torch.float32, device=DEV)
    kda.kda_chunk_fwd(q, k, v, g, beta, o, scale=inp.scale, initial_state=s0, final_state=fs,
                      cu_seqlens=cu, workspace=workspace, segment_chunks=L)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    return f64(o), f64(fs)


def oracle(inp):
    s0 = None if inp.initial_state is None else state_from_abi(inp.initial_state)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy()
    o, S = kda_recurrent(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.scale, s0, cu)
    return o, state_to_abi(S)


# Chunks per sequence 11, 0, 1, 8, 1, 3, 16: with L = 3 the first is cut into
# segments of 2, 3, 3, 3 chunks, the fourth into 2, 3, 3, the last into
# 2, 3, 3, 2, 3, 3; the others stay whole.
LENGTHS = [700, 0, 1, 450, 64, 129, 1000]


@pytest.mark.parametrize("L", [1, 2, 3, 5, 16, 0])
def test_segmented_parity_varlen(kda, L):
    inp = W.random_prefill(60, sum(LENGTHS), 3, 128, s0_std=0.1, lengths=LENGTHS,
                           g_fn=lambda z: -5.0 * torch.sigmoid(z - 3.0))
    inp.scale = 0.5
    o, S = run_seg(kda, inp, L)
    o_ref, S_ref = oracle(inp)
    assert rel_max(o, o_ref) <= TOL_BF16
    assert rel_fro(S, S_ref) <= TOL_STATE


@pytest.mark.parametrize("g_fn", [lambda z: -5.0 * torch.sigmoid(z),
                                  lambda z: torch.zeros_like(z),
                                  lambda z: torch.full_like(z, -5.0)],
                         ids=["k3_decay", "no_decay", "saturated_decay"])
def test_segmented_single_sequence_without_cu(kda, g_fn):
    """cu_seqlens NULL (the index pass still runs to number the segments);
    1300 tokens = 21 chunks, the last one ragged, in 11 segments of 1 or 2."""
    inp = W.random_prefill(61, 1300, 2, 128, s0_std=0.3, g_fn=g_fn)
    assert inp.cu_seqlens is None
    o, S = run_seg(kda, inp, 2)
    o_ref, S_ref = oracle(inp)
    assert rel_max(o, o_ref) <= TOL_BF16
    assert rel_fro(S, S_ref) <= TOL_STATE


def test_segmented_zero_initial_state(kda):
    inp = W.random_prefill(62, 900, 2, 128, s0_std=0.0, lengths=[900])
    inp.initial_state = None
    o, S = run_seg(kda, inp, 3)
    o_ref, S_ref = oracle(inp)
    assert rel_max(o, o_ref) <= TOL_BF16
    assert rel_fro(S, S_ref) <= TOL_STATE


@pytest.mark.parametrize("L", [1, 4])
def test_segmented_final_state_in_place(kda, L):
    """final_state aliasing initial_state: the output pass reads a split
    sequence's initial state from the copy the transition pass took, so the
    last segment may overwrite it while the first has not started."""
    inp = W.random_prefill(63, 1500, 2, 128, s0_std=0.2, lengths=[1200, 300],
                           g_fn=lambda z: -5.0 * torch.sigmoid(z - 5.0))
    o, S = run_seg(kda, inp, L, in_place=True)
    o_ref, S_ref = oracle(inp)
    assert rel_max(o, o_ref) <= TOL_BF16
    assert rel_fro(S, S_ref) <= TOL_STATE


def test_segmented_agrees_with_whole_sequences(kda):
    """Split and unsplit state passes round the same operands except the
    entry states of the segments (composed in fp32 from maps built with fp16
    state operands): far inside the bf16 bound of each other."""
    inp = W.random_prefill(64, 2500, 4, 128, s0_std=0.05, lengths=[2500],
                           g_fn=lambda z: -5.0 * torch.sigmoid(z - 2.0))
    o0, S0 = run_seg(kda, inp, 0)
    for L in (1, 3, 8):
        o, S = run_seg(kda, inp, L)
        assert rel_max(o, o0) <= 0.25 * TOL_BF16
        assert rel_fro(S, S0) <= 0.1 * TOL_STATE


def test_segmented_dirty_workspace_is_deterministic(kda):
    inp = W.random_prefill(65, 1100, 3, 128, s0_std=0.05, lengths=[129, 0, 900, 71])
    N, T, H = inp.N, inp.T, inp.H
    nbytes = kda.kda_chunk_fwd_segmented_workspace_bytes(N, T, H, 128, 128, 64, torch.bfloat16, 2)
    ws = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device=DEV)
    o1, S1 = run_seg(kda, inp, 2, workspace=ws)
    o2, S2 = run_seg(kda, inp, 2, workspace=ws)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)
    o_ref, S_ref = oracle(inp)
    assert rel_max(o1, o_ref) <= TOL_BF16
    assert rel_fro(S1, S_ref) <= TOL_STATE


def test_segmented_malformed_cu_seqlens_sets_status_without_fault(kda):
    inp = W.random_prefill(66, 512, 2, 128, lengths=[300, 212])
    q, k, v = inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV)
    bad = torch.tensor([0, 400, 300], dtype=torch.int32, device=DEV)
    o = torch.zeros((inp.T, 2, 128), device=DEV)
    fs = torch.empty((2, 2, 128, 128), device=DEV)
    kda.kda_chunk_fwd(q, k, v, inp.g.to(DEV), inp.beta.to(DEV), o, final_state=fs,
                      cu_seqlens=bad, segment_chunks=2)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == kda.KDA_ERR_DEVICE_BOUNDS
    assert kda.kda_get_device_status() == 0   # reading clears it


def test_auto_split_gated_matches_oracle(kda):
    """The gated entry point picks its segment length itself (here 4 chunks:
    one 2000-token sequence, 2 heads): gate, then the recurrence."""
    inp = W.random_prefill(67, 2000, 2, 128, s0_std=0.05, lengths=[2000])
    T, H, D = inp.T, inp.H, 128
    assert kda.kda_chunk_fwd_segment_chunks(1, T, H) == 4
    r = torch.Generator().manual_seed(68)
    g_raw = torch.randn((T, H, D), generator=r).to(torch.bfloat16)
    A_log = 0.5 * torch.randn((H,), generator=r)
    dt_bias = torch.randn((H, D), generator=r)
    g = gate(g_raw, A_log.numpy(), dt_bias.numpy(), -5.0)
    o = torch.empty((T, H, D), device=DEV)
    fs = torch.empty((1, H, D, D), device=DEV)
    kda.kda_chunk_fwd_gated(inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV), g_raw.to(DEV),
                            inp.beta.to(DEV), o, A_log=A_log.to(DEV), dt_bias=dt_bias.to(DEV),
                            initial_state=inp.initial_state.to(DEV), final_state=fs,
                            cu_seqlens=inp.cu_seqlens.to(DEV))
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    o_ref, S_ref = kda_recurrent(inp.q, inp.k, inp.v, g, inp.beta, 1.0,
                                 state_from_abi(inp.initial_state), inp.cu_seqlens.numpy())
    assert rel_max(f64(o), o_ref) <= TOL_BF16
    assert rel_fro(f64(fs), state_to_abi(S_ref)) <= TOL_STATE
