"""GPU parity: every libkda kernel against the float64 oracle, through the C ABI.

Tolerances (stated by the workloads): outputs max|delta| / RMS(reference)
<= 1e-4 for float32 activations and <= 2e-2 for bfloat16 activations; final
state relative Frobenius error <= 1e-2.  Full-size workloads run in the launch
configuration the benchmark times and are compared on sampled heads or
sequences that the oracle recomputes from regenerated input slabs.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import (kda_decode_step as o_decode, kda_recurrent, prologue as o_prologue,
                    state_from_abi, state_to_abi)

pytestmark = pytest.mark.gpu

TOL_F32, TOL_BF16, TOL_STATE = 1e-4, 2e-2, 1e-2


@pytest.fixture(scope="module")
def kda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import gated_delta_rule_prologue_b200 as m
    return m


def rel_max(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got))
    return float(np.max(np.abs(got - ref)) / np.sqrt(np.mean(ref * ref)))


def rel_fro(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got))
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


# Unit roundoff of each storage type: rounding to nearest moves a value by at
# most this fraction of itself (bf16: 8 significant bits, fp16: 11).
UNIT_ROUNDOFF = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}


def check_rounded(got, ref, dtype):
    """Elementwise check of a stored activation: the rounding of the storage
    type plus float32 arithmetic noise (1e-5 of the RMS)."""
    rms = np.sqrt(np.mean(ref * ref))
    if dtype in UNIT_ROUNDOFF:
        assert np.all(np.abs(f64(got) - ref) <= UNIT_ROUNDOFF[dtype] * np.abs(ref) + 1e-5 * rms)
    else:
        assert rel_max(f64(got), ref) <= 1e-5


# kda_chunk_fwd's two ways through the tensor-core path: the two-pass kernels
# with a scratch workspace (the default) and the one-pass kernel.
PASSES = {"two_pass": "auto", "one_pass": None}


def run_chunk(kda, inp, *, chunk=None, in_place=False, workspace="auto"):
    dev = "cuda"
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    g, beta = inp.g.to(dev), inp.beta.to(dev)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(dev)
    N, H, D = inp.N, inp.H, inp.q.shape[2]
    s0 = None if inp.initial_state is None else inp.initial_state.to(dev).contiguous()
    fs = s0 if (in_place and s0 is not None) else torch.empty((N, H, D, D), device=dev)
    o = torch.empty(v.shape, dtype=torch.float32, device=dev)
    kda.kda_chunk_fwd(q, k, v, g, beta, o, scale=inp.scale, initial_state=s0, final_state=fs,
                      cu_seqlens=cu, chunk=chunk or inp.chunk, workspace=workspace)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    return f64(o), f64(fs)


def oracle_chunk(inp):
    s0 = None if inp.initial_state is None else state_from_abi(inp.initial_state)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy()
    o, S = kda_recurrent(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.scale, s0, cu)
    return o, state_to_abi(S)


# --- chunk_fwd ---------------------------------------------------------------

def test_tiny_f32_parity(kda):
    inp = W.tiny_f32()
    o, S = run_chunk(kda, inp)
    o_ref, S_ref = oracle_chunk(inp)
    assert rel_max(o, o_ref) <= TOL_F32
    assert rel_fro(S, S_ref) <= 1e-5


@pytest.mark.parametrize("passes", list(PASSES))
def test_seq4k_bf16_parity(kda, passes):
    inp = W.seq4k_bf16()
    o, S = run_chunk(kda, inp, workspace=PASSES[passes])
    o_ref, S_ref = oracle_chunk(inp)
    assert rel_max(o, o_ref) <= TOL_BF16
    assert rel_fro(S, S_ref) <= TOL_STATE


EDGE = [
    # (name, D, chunk, bf16, lengths, g_shift, s0_std, g_fn)
    ("ragged_f32_d128_c64", 128, 64, False, [200, 1, 64, 0, 63, 130], 0.0, 0.3, None),
    ("ragged_bf16_d128_c64", 128, 64, True, [200, 1, 64, 0, 63, 130], 0.0, 0.3, None),
    ("bf16_d64_c32", 64, 32, True, [77, 150], 0.0, 0.1, None),
    ("f32_d32_c16", 32, 16, False, [33, 5], 0.0, 0.1, None),
    ("bf16_d16_c64", 16, 64, True, [100], 0.0, 0.0, None),
    ("slow_decay_bf16", 128, 64, True, [700], 0.0, 0.05,
     lambda z: -5.0 * torch.sigmoid(z - 6.0)),
    ("saturated_decay_bf16", 128, 64, True, [300], 0.0, 0.05,
     lambda z: torch.full_like(z, -5.0)),
    ("no_decay_bf16", 128, 64, True, [190], 0.0, 0.05, lambda z: torch.zeros_like(z)),
]


@pytest.mark.parametrize("passes", list(PASSES))
@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_chunk_edge_cases(kda, case, passes):
    name, D, chunk, bf16, lengths, g_shift, s0_std, g_fn = case
    if passes == "one_pass" and not (bf16 and D == 128 and chunk == 64):
        pytest.skip("only the tensor-core path has two variants")
    inp = W.random_prefill(100 + EDGE.index(case), sum(lengths), 3, D, bf16=bf16,
                           g_shift=g_shift, s0_std=s0_std, lengths=lengths, chunk=chunk,
                           g_fn=g_fn)
    inp.scale = 0.5
    o, S = run_chunk(kda, inp, workspace=PASSES[passes])
    o_ref, S_ref = oracle_chunk(inp)
    tol = TOL_BF16 if bf16 else TOL_F32
    assert rel_max(o, o_ref) <= tol
    assert rel_fro(S, S_ref) <= (TOL_STATE if bf16 else 1e-5)


@pytest.mark.parametrize("passes", list(PASSES))
def test_chunk_final_state_in_place(kda, passes):
    inp = W.random_prefill(5, 150, 2, 128, s0_std=0.1, lengths=[90, 60],
                           g_fn=lambda z: -5.0 * torch.sigmoid(z - 5.0))
    o, S = run_chunk(kda, inp, in_place=True, workspace=PASSES[passes])
    o_ref, S_ref = oracle_chunk(inp)
    assert rel_max(o, o_ref) <= TOL_BF16
    assert rel_fro(S, S_ref) <= TOL_STATE


def test_chunk_size_does_not_change_results(kda):
    inp = W.random_prefill(6, 257, 2, 64, bf16=False, s0_std=0.1,
                           g_fn=lambda z: -5.0 * torch.sigmoid(z - 4.0))
    outs = [run_chunk(kda, inp, chunk=c) for c in (16, 32, 64)]
    for o, S in outs[1:]:
        assert rel_max(o, outs[0][0]) <= 1e-4
        assert rel_fro(S, outs[0][1]) <= 1e-5


def test_tensor_core_and_cuda_core_paths_agree(kda):
    """bf16, d=128: chunk 64 runs the tcgen05 kernels (two-pass and one-pass),
    chunk 32 the fp32 CUDA-core kernel; all within the bf16 bound of each
    other, and the two tensor-core variants, which round the same operands,
    much closer than that."""
    inp = W.random_prefill(9, 333, 2, 128, s0_std=0.1, lengths=[200, 133],
                           g_fn=lambda z: -5.0 * torch.sigmoid(z - 1.0))
    o_tc, S_tc = run_chunk(kda, inp, chunk=64)
    o_1p, S_1p = run_chunk(kda, inp, chunk=64, workspace=None)
    o_cc, S_cc = run_chunk(kda, inp, chunk=32)
    assert rel_max(o_tc, o_cc) <= TOL_BF16
    assert rel_fro(S_tc, S_cc) <= TOL_STATE
    assert rel_max(o_1p, o_cc) <= TOL_BF16
    assert rel_max(o_tc, o_1p) <= 0.25 * TOL_BF16
    assert rel_fro(S_tc, S_1p) <= 0.1 * TOL_STATE


def test_two_pass_many_ragged_sequences(kda):
    """20 sequences x 4 heads through the two-pass path: empty sequences,
    shorter than a chunk, exact multiples of 64, several chunks; the chunk
    index, the record walk and the per-sequence state hand-off."""
    lengths = [0, 1, 63, 64, 65, 128, 200, 7, 300, 129, 64, 0, 31, 190, 256, 2, 77, 140, 95, 33]
    inp = W.random_prefill(14, sum(lengths), 4, 128, s0_std=0.1, lengths=lengths,
                           g_fn=lambda z: -5.0 * torch.sigmoid(z - 4.0))
    o, S = run_chunk(kda, inp)
    o_ref, S_ref = oracle_chunk(inp)
    assert rel_max(o, o_ref) <= TOL_BF16
    assert rel_fro(S, S_ref) <= TOL_STATE
    o1, S1 = run_chunk(kda, inp, workspace=None)
    assert rel_max(o, o1) <= 0.25 * TOL_BF16


def test_two_pass_workspace_reuse_is_deterministic(kda):
    """The same caller-owned workspace twice in a row, dirty from the first
    call: bit-identical results."""
    inp = W.random_prefill(12, 500, 4, 128, s0_std=0.05, lengths=[129, 0, 64, 307],
                           g_fn=lambda z: -5.0 * torch.sigmoid(z - 3.0))
    N, T, H = inp.N, inp.T, inp.H
    nbytes = kda.kda_chunk_fwd_workspace_bytes(N, T, H, 128, 128, 64, torch.bfloat16)
    assert nbytes > 0
    ws = torch.full((nbytes,), 0xA5, dtype=torch.uint8, device="cuda")
    o1, S1 = run_chunk(kda, inp, workspace=ws)
    o2, S2 = run_chunk(kda, inp, workspace=ws)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)
    o_ref, S_ref = oracle_chunk(inp)
    assert rel_max(o1, o_ref) <= TOL_BF16
    assert rel_fro(S1, S_ref) <= TOL_STATE


def test_two_pass_malformed_cu_seqlens_sets_status_without_fault(kda):
    inp = W.random_prefill(13, 256, 2, 128, lengths=[100, 156])
    dev = "cuda"
    bad = torch.tensor([0, 300, 20], dtype=torch.int32, device=dev)  # past T, then decreasing
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    o = torch.empty(v.shape, dtype=torch.float32, device=dev)
    kda.kda_chunk_fwd(q, k, v, inp.g.to(dev), inp.beta.to(dev), o, cu_seqlens=bad)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == kda.KDA_ERR_DEVICE_BOUNDS
    o2, _ = run_chunk(kda, inp)
    assert np.all(np.isfinite(o2))


def test_malformed_cu_seqlens_sets_status_without_fault(kda):
    inp = W.random_prefill(7, 64, 1, 16, bf16=False, lengths=[30, 34], chunk=16)
    dev = "cuda"
    bad = torch.tensor([0, 40, 20], dtype=torch.int32, device=dev)  # decreasing
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    o = torch.empty(v.shape, dtype=torch.float32, device=dev)
    kda.kda_chunk_fwd(q, k, v, inp.g.to(dev), inp.beta.to(dev), o, cu_seqlens=bad, chunk=16)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == kda.KDA_ERR_DEVICE_BOUNDS
    assert kda.kda_get_device_status() == 0    # cleared by the read
    o2, _ = run_chunk(kda, inp)                 # the context is still usable
    assert np.all(np.isfinite(o2))


# --- prologue ----------------------------------------------------------------

@pytest.mark.parametrize("dtype,out_dtype,D", [(torch.bfloat16, torch.bfloat16, 128),
                                               (torch.bfloat16, torch.float32, 128),
                                               (torch.bfloat16, torch.float16, 128),
                                               (torch.float32, torch.float32, 16),
                                               (torch.float32, torch.bfloat16, 64)])
def test_prologue_parity_varlen_with_cache(kda, dtype, out_dtype, D):
    H = 3
    lengths = [70, 0, 1, 2, 45, 33]
    T, N, C = sum(lengths), len(lengths), 3 * H * D
    r = torch.Generator().manual_seed(D)
    x = torch.randn((T, C), generator=r).to(dtype)
    w = 0.5 * torch.randn((C, 4), generator=r)
    cache = torch.randn((N, 3, C), generator=r).to(dtype)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    dev = "cuda"
    q = torch.empty((T, H, D), dtype=out_dtype, device=dev)
    k, v = torch.empty_like(q), torch.empty_like(q)
    cache_out = torch.empty((N, 3, C), dtype=dtype, device=dev)
    kda.kda_prologue(x.to(dev), w.to(dev), q, k, v, H=H, D=D, cache_in=cache.to(dev),
                     cache_out=cache_out, cu_seqlens=cu.to(dev))
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    q_ref, k_ref, v_ref, c_ref = o_prologue(x, w, H, D, cu.numpy(), cache)
    for got, ref in ((q, q_ref), (k, k_ref), (v, v_ref)):
        check_rounded(got, ref, out_dtype)
    np.testing.assert_array_equal(f64(cache_out), c_ref)   # a copy of inputs: exact


# --- full-size workloads, sampled ------------------------------------------------

def test_k3_prefill_full_size_sampled_heads(kda):
    """Fused prologue + chunkwise prefill over 32768 tokens x 96 heads, both the
    two-pass launch (the benchmark's) and the one-pass kernel; heads 0, 53 and
    95 recomputed by the oracle over all tokens."""
    inp = W.k3_prefill()
    T, H, D = inp.T, inp.H, inp.D
    dev = "cuda"
    x, w, g, beta = inp.x.to(dev), inp.conv_w.to(dev), inp.g.to(dev), inp.beta.to(dev)
    runs = {}
    for passes, ws in PASSES.items():
        o = torch.empty((T, H, D), dtype=torch.float32, device=dev)
        fs = torch.empty((1, H, D, D), device=dev)
        cache = torch.empty((1, 3, 3 * H * D), dtype=torch.bfloat16, device=dev)
        kda.kda_prologue_chunk_fwd(x, w, g, beta, o, H=H, D=D, scale=inp.scale, final_state=fs,
                                   cache_out=cache, workspace=ws)
        torch.cuda.synchronize()
        assert kda.kda_get_device_status() == 0
        np.testing.assert_array_equal(f64(cache[0]), f64(inp.x[-3:]))
        runs[passes] = (o.cpu(), fs.cpu())
        del o
        torch.cuda.empty_cache()
    del x, g, beta
    for h in (0, 53, 95):
        xh, wh, gh, bh = W.k3_prefill_head(h)
        qr, kr, vr, _ = o_prologue(xh.reshape(T, 3 * D), wh.reshape(3 * D, 4), 1, D)
        o_ref, S_ref = kda_recurrent(qr, kr, vr, gh[:, None, :], bh[:, None], inp.scale)
        for passes, (o, fs) in runs.items():
            assert rel_max(f64(o[:, h]), o_ref[:, 0]) <= TOL_BF16, passes
            assert rel_fro(f64(fs[0, h]), state_to_abi(S_ref)[0, 0]) <= TOL_STATE, passes


def test_k3_unfused_full_size_sampled_heads(kda):
    """kda_prologue (fp16 q/k/v) followed by kda_chunk_fwd over the full K3
    workload; heads 3 and 61 against the oracle."""
    inp = W.k3_prefill()
    T, H, D = inp.T, inp.H, inp.D
    dev = "cuda"
    q = torch.empty((T, H, D), dtype=torch.float16, device=dev)
    k, v = torch.empty_like(q), torch.empty_like(q)
    kda.kda_prologue(inp.x.to(dev), inp.conv_w.to(dev), q, k, v, H=H, D=D)
    o = torch.empty((T, H, D), dtype=torch.float32, device=dev)
    fs = torch.empty((1, H, D, D), device=dev)
    kda.kda_chunk_fwd(q, k, v, inp.g.to(dev), inp.beta.to(dev), o, scale=inp.scale,
                      final_state=fs, chunk=inp.chunk)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    for h in (3, 61):
        xh, wh, gh, bh = W.k3_prefill_head(h)
        qr, kr, vr, _ = o_prologue(xh.reshape(T, 3 * D), wh.reshape(3 * D, 4), 1, D)
        o_ref, S_ref = kda_recurrent(qr, kr, vr, gh[:, None, :], bh[:, None], inp.scale)
        assert rel_max(f64(o[:, h]), o_ref[:, 0]) <= TOL_BF16
        assert rel_fro(f64(fs[0, h]), state_to_abi(S_ref)[0, 0]) <= TOL_STATE


def test_k3_prologue_kernel_full_size_sampled_heads(kda):
    """The standalone prologue over the full K3-shaped input, fp16 outputs."""
    inp = W.k3_prefill()
    T, H, D = inp.T, inp.H, inp.D
    dev = "cuda"
    q = torch.empty((T, H, D), dtype=torch.float16, device=dev)
    k, v = torch.empty_like(q), torch.empty_like(q)
    kda.kda_prologue(inp.x.to(dev), inp.conv_w.to(dev), q, k, v, H=H, D=D)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    for h in (7, 88):
        xh, wh, _, _ = W.k3_prefill_head(h)
        qr, kr, vr, _ = o_prologue(xh.reshape(T, 3 * D), wh.reshape(3 * D, 4), 1, D)
        for got, ref in ((q[:, h], qr[:, 0]), (k[:, h], kr[:, 0]), (v[:, h], vr[:, 0])):
            check_rounded(got, ref, torch.float16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("passes", list(PASSES))
@pytest.mark.parametrize("lengths", [([70, 1, 130, 64], [5, 100, 2, 66]),
                                     ([70, 0, 130, 1, 200], [0, 100, 2, 66, 3])],
                         ids=["nonempty", "with_empty"])
def test_fused_prefill_varlen_with_cache_and_resume(kda, dtype, passes, lengths):
    """Fused path over packed sequences with conv cache and initial state in,
    cache and final state out; then a second call continuing every sequence
    from the first call's cache and state.  Both calls match the oracle run
    over the concatenated tokens; a sequence that is empty in a call passes
    its cache and state through."""
    dev = "cuda"
    H, D = 2, 128
    l1, l2 = lengths
    N, C = len(l1), 3 * H * D
    r = torch.Generator().manual_seed(31)
    xs = [torch.randn((a + b, C), generator=r).to(dtype) for a, b in zip(l1, l2)]
    w = 0.5 * torch.randn((C, 4), generator=r)
    gs = [-5.0 * torch.sigmoid(torch.randn((a + b, H, D), generator=r) - 2.0) for a, b in zip(l1, l2)]
    bs = [torch.sigmoid(torch.randn((a + b, H), generator=r)) for a, b in zip(l1, l2)]
    cache0 = torch.randn((N, 3, C), generator=r).to(dtype)
    s0 = 0.05 * torch.randn((N, H, D, D), generator=r)

    def pack(lists, part):
        return torch.cat([t[:a] if part == 0 else t[a:] for t, a in zip(lists, l1)]).contiguous()

    outs = []
    cache_in, state = cache0.to(dev), s0.to(dev)
    for part, lens in ((0, l1), (1, l2)):
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
        T = sum(lens)
        o = torch.empty((T, H, D), dtype=torch.float32, device=dev)
        cache_out = torch.empty((N, 3, C), dtype=dtype, device=dev)
        fs = torch.empty((N, H, D, D), device=dev)
        kda.kda_prologue_chunk_fwd(pack(xs, part).to(dev), w.to(dev), pack(gs, part).to(dev),
                                   pack(bs, part).to(dev), o, H=H, D=D, cache_in=cache_in,
                                   cache_out=cache_out, initial_state=state, final_state=fs,
                                   cu_seqlens=cu, workspace=PASSES[passes])
        outs.append((o, cu))
        cache_in, state = cache_out, fs
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    lens_all = [a + b for a, b in zip(l1, l2)]
    cu_all = np.concatenate([[0], np.cumsum(lens_all)])
    qr, kr, vr, c_ref = o_prologue(torch.cat(xs), w, H, D, cu_all, cache0)
    o_ref, S_ref = kda_recurrent(qr, kr, vr, torch.cat(gs), torch.cat(bs), 1.0,
                                 state_from_abi(s0), cu_all)
    got = np.zeros_like(o_ref)
    for n in range(N):
        a = cu_all[n]
        got[a:a + l1[n]] = f64(outs[0][0])[int(outs[0][1][n]):int(outs[0][1][n + 1])]
        got[a + l1[n]:a + lens_all[n]] = f64(outs[1][0])[int(outs[1][1][n]):int(outs[1][1][n + 1])]
    assert rel_max(got, o_ref) <= TOL_BF16
    assert rel_fro(f64(state), state_to_abi(S_ref)) <= TOL_STATE
    np.testing.assert_array_equal(f64(cache_in), c_ref)


def test_fused_and_unfused_prefill_agree(kda):
    """kda_prologue_chunk_fwd equals kda_prologue (fp16 hand-off) followed by
    kda_chunk_fwd within the bf16 bound."""
    dev = "cuda"
    T, H, D = 400, 3, 128
    C = 3 * H * D
    r = torch.Generator().manual_seed(41)
    x = torch.randn((T, C), generator=r).to(torch.bfloat16).to(dev)
    w = (0.5 * torch.randn((C, 4), generator=r)).to(dev)
    g = (-5.0 * torch.sigmoid(torch.randn((T, H, D), generator=r))).to(dev)
    beta = torch.sigmoid(torch.randn((T, H), generator=r)).to(dev)
    o1 = torch.empty((T, H, D), dtype=torch.float32, device=dev)
    kda.kda_prologue_chunk_fwd(x, w, g, beta, o1, H=H, D=D)
    q, k, v, _ = _prefill_gpu(kda, x, w, H, D, act=torch.float16)
    o2 = torch.empty((T, H, D), dtype=torch.float32, device=dev)
    kda.kda_chunk_fwd(q, k, v, g, beta, o2)
    torch.cuda.synchronize()
    assert rel_max(f64(o1), f64(o2)) <= 2 * TOL_BF16


def test_varlen16_full_size_sampled(kda):
    inp = W.varlen16()
    o, S = run_chunk(kda, inp)
    lengths = W.varlen16_lengths()
    cu = np.concatenate([[0], np.cumsum(lengths)])
    picks = [(int(np.argmin(lengths)), 0), (int(np.argmax(lengths)), 31), (5, 17)]
    for n, h in picks:
        qn, kn, vn, gn, bn, s0 = W.varlen16_seq_head(n, h)
        o_ref, S_ref = kda_recurrent(qn[:, None], kn[:, None], vn[:, None], gn[:, None],
                                     bn[:, None], 1.0, state_from_abi(s0)[None, None])
        assert rel_max(o[cu[n]:cu[n + 1], h], o_ref[:, 0]) <= TOL_BF16
        assert rel_fro(S[n, h], state_to_abi(S_ref)[0, 0]) <= TOL_STATE


def test_decode256_full_size_sampled(kda):
    """256 x 96 heads, 3 consecutive in-place steps; sequences 0, 77, 255 checked."""
    steps = 3
    inp = W.decode256(steps=steps)
    dev = "cuda"
    H, D = inp.H, inp.D
    state = inp.state.to(dev)
    cache = inp.conv_cache.to(dev)
    w = inp.conv_w.to(dev)
    outs = []
    for s in range(steps):
        o = torch.empty((inp.N, H, D), dtype=torch.float32, device=dev)
        kda.kda_decode_step(inp.x[s].to(dev), w, cache, inp.g[s].to(dev), inp.beta[s].to(dev),
                            state, o, H=H, D=D, scale=inp.scale)
        outs.append(o)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    ns = [0, 77, 255]
    st0, c0, xs, gs, bs, wr = W.decode256_seqs(ns, steps)
    S = state_from_abi(st0)
    c = c0
    for s in range(steps):
        o_ref, S, c = o_decode(xs[s], wr, c, gs[s], bs[s], S, H, D)
        assert rel_max(f64(outs[s][ns]), o_ref) <= TOL_BF16
    assert rel_fro(f64(state[ns]), state_to_abi(S)) <= TOL_STATE
    np.testing.assert_array_equal(f64(cache[ns]), c)


# --- cross-checks between GPU paths ------------------------------------------------

def _prefill_gpu(kda, x, w, H, D, cache_in=None, s0=None, cu=None, act=torch.float32):
    dev = "cuda"
    T = x.shape[0]
    N = 1 if cu is None else cu.numel() - 1
    q = torch.empty((T, H, D), dtype=act, device=dev)
    k, v = torch.empty_like(q), torch.empty_like(q)
    cache_out = torch.empty((N, 3, 3 * H * D), dtype=x.dtype, device=dev)
    kda.kda_prologue(x, w, q, k, v, H=H, D=D, cache_in=cache_in, cache_out=cache_out,
                     cu_seqlens=cu)
    return q, k, v, cache_out


def test_decode_kernel_matches_prologue_plus_chunk_kernel(kda):
    """Two independent GPU paths over the same tokens: prefill (prologue kernel
    + chunk kernel) and the decode kernel applied token by token."""
    dev = "cuda"
    N, T, H, D = 3, 40, 4, 128
    C = 3 * H * D
    r = torch.Generator().manual_seed(11)
    x = torch.randn((N, T, C), generator=r).to(torch.bfloat16)
    w = 0.5 * torch.randn((C, 4), generator=r)
    g = -5.0 * torch.sigmoid(torch.randn((N, T, H, D), generator=r) - 3.0)
    beta = torch.sigmoid(torch.randn((N, T, H), generator=r))
    s0 = 0.05 * torch.randn((N, H, D, D), generator=r)
    cu = torch.arange(0, N * T + 1, T, dtype=torch.int32, device=dev)
    q, k, v, cache_out = _prefill_gpu(kda, x.reshape(N * T, C).to(dev), w.to(dev), H, D, cu=cu)
    o_pre = torch.empty(v.shape, dtype=torch.float32, device=dev)
    S_pre = torch.empty((N, H, D, D), device=dev)
    kda.kda_chunk_fwd(q, k, v, g.reshape(N * T, H, D).to(dev), beta.reshape(N * T, H).to(dev),
                      o_pre, initial_state=s0.to(dev), final_state=S_pre, cu_seqlens=cu)
    state = s0.to(dev).clone()
    cache = torch.zeros((N, 3, C), dtype=torch.bfloat16, device=dev)
    o_dec = torch.empty((N, T, H, D), dtype=torch.float32, device=dev)
    for t in range(T):
        ot = torch.empty((N, H, D), dtype=torch.float32, device=dev)
        kda.kda_decode_step(x[:, t].contiguous().to(dev), w.to(dev), cache,
                            g[:, t].contiguous().to(dev), beta[:, t].contiguous().to(dev),
                            state, ot, H=H, D=D)
        o_dec[:, t] = ot
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    assert rel_max(f64(o_pre).reshape(N, T, H, D), f64(o_dec)) <= 1e-4
    assert rel_fro(f64(S_pre), f64(state)) <= 1e-5
    np.testing.assert_array_equal(f64(cache), f64(cache_out))


@pytest.mark.parametrize("act", [torch.float32, torch.float16])
def test_resume_prefill_with_state_and_cache_handoff(kda, act):
    """Prefill [0, T1) then [T1, T) with final_state / conv cache handed over:
    both halves match the oracle's single pass over [0, T) (float32 hand-off:
    CUDA-core chunk kernel; float16 hand-off: tensor-core chunk kernel)."""
    dev = "cuda"
    T, T1, H, D = 300, 131, 2, 128
    C = 3 * H * D
    r = torch.Generator().manual_seed(12)
    x = torch.randn((T, C), generator=r).to(torch.bfloat16)
    w = 0.5 * torch.randn((C, 4), generator=r)
    g = -5.0 * torch.sigmoid(torch.randn((T, H, D), generator=r) - 4.0)
    beta = torch.sigmoid(torch.randn((T, H), generator=r))
    xd, wd, gd, bd = x.to(dev), w.to(dev), g.to(dev), beta.to(dev)
    q1, k1, v1, c1 = _prefill_gpu(kda, xd[:T1].contiguous(), wd, H, D, act=act)
    S1 = torch.empty((1, H, D, D), device=dev)
    o1 = torch.empty(v1.shape, dtype=torch.float32, device=dev)
    kda.kda_chunk_fwd(q1, k1, v1, gd[:T1].contiguous(), bd[:T1].contiguous(), o1, final_state=S1)
    q2, k2, v2, _ = _prefill_gpu(kda, xd[T1:].contiguous(), wd, H, D, cache_in=c1, act=act)
    o2 = torch.empty(v2.shape, dtype=torch.float32, device=dev)
    S2 = torch.empty((1, H, D, D), device=dev)
    kda.kda_chunk_fwd(q2, k2, v2, gd[T1:].contiguous(), bd[T1:].contiguous(), o2,
                      initial_state=S1, final_state=S2)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    qr, kr, vr, _ = o_prologue(x, w, H, D)
    o_ref, S_ref = kda_recurrent(qr, kr, vr, g, beta, 1.0)
    tol = TOL_BF16 if act != torch.float32 else TOL_F32
    assert rel_max(f64(torch.cat([o1, o2])), o_ref) <= tol
    assert rel_fro(f64(S2), state_to_abi(S_ref)) <= (TOL_STATE if act != torch.float32 else 1e-5)
