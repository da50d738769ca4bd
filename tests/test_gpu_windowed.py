"""GPU checks of the windowed two-pass prefill (kda_chunk_fwd_windowed_ws).

The in-chunk work of a chunk does not depend on the carried state
("KimiK3轻量化复刻实现KDA并行解析，Chunkwise并行与状态压缩机制详解", Figure 1),
so the prep pass can run a window of chunks ahead of the state pass and the
workspace only has to hold one window's records.  The windowed call performs
the same arithmetic in the same order as the unsplit two-pass call
(kda_chunk_fwd_segmented_ws with segment_chunks = 0), so outputs and final
states must agree bit for bit: windows of one chunk, windows that cut
sequences anywhere (including inside a sequence's first and last chunks'
neighbours), windows past the last chunk, empty sequences and an in-place
final state.  One case is also compared with the float64 oracle.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import kda_recurrent, state_from_abi, state_to_abi

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


def run(kda, inp, *, window=None, in_place=False, workspace="auto"):
    q, k, v = inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV)
    g, beta = inp.g.to(DEV), inp.beta.to(DEV)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(DEV)
    N, H, D = inp.N, inp.H, inp.q.shape[2]
    s0 = None if inp.initial_state is None else inp.initial_state.to(DEV).contiguous()
    fs = s0 if (in_place and s0 is not None) else torch.empty((N, H, D, D), device=DEV)
    o = torch.full(v.shape, float("nan"), dtype=torch.float32, device=DEV)
    if window is None:
        kda.kda_chunk_fwd(q, k, v, g, beta, o, scale=inp.scale, initial_state=s0,
                          final_state=fs, cu_seqlens=cu, segment_chunks=0)
    else:
        kda.kda_chunk_fwd(q, k, v, g, beta, o, scale=inp.scale, initial_state=s0,
                          final_state=fs, cu_seqlens=cu, window_chunks=window,
                          workspace=workspace)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    return o.cpu(), fs.cpu()


# Chunks per sequence: 11, 0, 1, 3, 1, 0, 16, 1 (42 in all, capacity 8 + 35 = 43).
LENGTHS = [700, 0, 1, 129, 64, 0, 1000, 37]


@pytest.mark.parametrize("window", [1, 2, 3, 7, 16, 43, 1000])
def test_windowed_matches_unsplit_varlen(kda, window):
    inp = W.random_prefill(71, sum(LENGTHS), 3, 128, s0_std=0.1, lengths=LENGTHS,
                           g_fn=lambda z: -5.0 * torch.sigmoid(z - 3.0))
    o_ref, s_ref = run(kda, inp)
    o, s = run(kda, inp, window=window)
    assert torch.equal(o, o_ref)
    assert torch.equal(s, s_ref)


@pytest.mark.parametrize("window", [1, 5, 64])
def test_windowed_single_sequence_without_cu(kda, window):
    inp = W.random_prefill(72, 4096 + 37, 4, 128, s0_std=0.1)
    o_ref, s_ref = run(kda, inp)
    o, s = run(kda, inp, window=window)
    assert torch.equal(o, o_ref)
    assert torch.equal(s, s_ref)


def test_windowed_in_place_final_state_and_oracle(kda):
    inp = W.random_prefill(73, sum(LENGTHS), 2, 128, s0_std=0.1, lengths=LENGTHS)
    o_ref, s_ref = run(kda, inp)
    o, s = run(kda, inp, window=4, in_place=True)
    assert torch.equal(o, o_ref)
    assert torch.equal(s, s_ref)
    ro, rS = kda_recurrent(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.scale,
                           state_from_abi(inp.initial_state), inp.cu_seqlens.numpy())
    rs = state_to_abi(rS)
    err = float(np.max(np.abs(f64(o) - ro)) / np.sqrt(np.mean(ro * ro)))
    assert err <= TOL_BF16, err
    ferr = float(np.linalg.norm(f64(s) - rs) / np.linalg.norm(rs))
    assert ferr <= TOL_STATE, ferr


def test_windowed_dirty_workspace_is_deterministic(kda):
    inp = W.random_prefill(74, sum(LENGTHS), 3, 128, s0_std=0.1, lengths=LENGTHS)
    N, T, H = inp.N, inp.q.shape[0], inp.H
    nbytes = kda.kda_chunk_fwd_windowed_workspace_bytes(N, T, H, 128, 128, 64, inp.q.dtype, 3)
    g = torch.Generator(device=DEV).manual_seed(5)
    ws = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, device=DEV, generator=g)
    first = run(kda, inp, window=3, workspace=ws)
    ws.random_(0, 256, generator=g)
    second = run(kda, inp, window=3, workspace=ws)
    assert torch.equal(first[0], second[0]) and torch.equal(first[1], second[1])


@pytest.mark.parametrize("window", [1, 3, 17])
def test_windowed_fused_matches_unsplit(kda, window):
    """The prologue inside the prep pass, one window at a time: read-out, final state and
    conv cache equal the two-pass fused call's.  Five sequences x 32 heads give 640 state
    chains, so the unwindowed call runs whole sequences too."""
    lengths = [300, 0, 1, 700, 129]
    H, D = 32, 128
    assert kda.lib.kda_chunk_fwd_segment_chunks(len(lengths), sum(lengths), H) == 0
    T, N, C = sum(lengths), len(lengths), 3 * H * D
    r = torch.Generator().manual_seed(75)
    x = torch.randn((T, C), generator=r).to(torch.bfloat16).to(DEV)
    w = (0.5 * torch.randn((C, 4), generator=r)).to(DEV)
    g = (-5.0 * torch.sigmoid(torch.randn((T, H, D), generator=r) - 3.0)).to(DEV)
    beta = torch.sigmoid(torch.randn((T, H), generator=r)).to(DEV)
    cache_in = torch.randn((N, 3, C), generator=r).to(torch.bfloat16).to(DEV)
    s0 = (0.1 * torch.randn((N, H, D, D), generator=r)).to(DEV)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32).to(DEV)
    outs = []
    for win in (None, window):
        o = torch.full((T, H, D), float("nan"), device=DEV)
        fs = torch.empty((N, H, D, D), device=DEV)
        cache_out = torch.empty_like(cache_in)
        kda.kda_prologue_chunk_fwd(x, w, g, beta, o, H=H, D=D, scale=0.5, cache_in=cache_in,
                                   cache_out=cache_out, initial_state=s0, final_state=fs,
                                   cu_seqlens=cu, window_chunks=win)
        torch.cuda.synchronize()
        assert kda.kda_get_device_status() == 0
        outs.append((o.cpu(), fs.cpu(), cache_out.cpu()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
