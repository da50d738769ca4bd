"""Pins for the oracle's prologue (short conv, SiLU, L2) and decode step.

Sources: [W1] "Kimi K3的线性注意力：从源码看懂KDA如何更新记忆", 第二站 (short conv
of width 4 that never looks ahead, SiLU inside the conv module, L2 on q and
k); [W4] "KimiK3轻量化复刻实现KDA并行解析，Chunkwise并行与状态压缩机制详解",
ShortConv paragraph (per channel, the current token and the three before it).
"""
import numpy as np
import torch
from scipy.signal import lfilter
from scipy.special import expit

from oracle import (L2_EPS, kda_decode_step, kda_recurrent, l2_normalize, prologue,
                    short_conv, silu)

R = np.random.default_rng(99)


def test_conv_equals_library_iir_filter_with_zero_history():
    """A causal FIR filter with taps w[c, 3], w[c, 2], w[c, 1], w[c, 0] on
    delays 0..3 is scipy's lfilter with b = w[c, ::-1] and zero initial state."""
    T, C = 37, 11
    x = R.standard_normal((T, C))
    w = R.standard_normal((C, 4))
    y, _ = short_conv(x, w)
    for c in range(C):
        np.testing.assert_allclose(y[:, c], lfilter(w[c, ::-1], [1.0], x[:, c]),
                                   rtol=1e-12, atol=1e-13)


def test_conv_with_cache_equals_library_filter_on_extended_input():
    T, C = 9, 5
    x = R.standard_normal((T, C))
    w = R.standard_normal((C, 4))
    cache = R.standard_normal((1, 3, C))
    y, cache_out = short_conv(x, w, cache_in=cache)
    ext = np.concatenate([cache[0], x])
    for c in range(C):
        np.testing.assert_allclose(y[:, c], lfilter(w[c, ::-1], [1.0], ext[:, c])[3:],
                                   rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(cache_out[0], x[-3:])


def test_conv_is_causal():
    """Changing tokens after t leaves every output at or before t unchanged."""
    T, C = 30, 8
    x = R.standard_normal((T, C))
    w = R.standard_normal((C, 4))
    y, _ = short_conv(x, w)
    for t in (0, 1, 2, 3, 17, 28):
        x2 = x.copy()
        x2[t + 1:] = R.standard_normal((T - t - 1, C))
        y2, _ = short_conv(x2, w)
        assert np.array_equal(y2[:t + 1], y[:t + 1])


def test_conv_never_crosses_sequence_boundaries():
    lengths = [4, 1, 2, 10]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    C = 6
    x = R.standard_normal((cu[-1], C))
    w = R.standard_normal((C, 4))
    cache = R.standard_normal((len(lengths), 3, C))
    y, cache_out = short_conv(x, w, cu, cache)
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        yn, cn = short_conv(x[a:b], w, None, cache[n:n + 1])
        assert np.array_equal(y[a:b], yn) and np.array_equal(cache_out[n], cn[0])
    # a one-token sequence keeps two cache rows in its new cache
    np.testing.assert_array_equal(cache_out[1], np.concatenate([cache[1][1:], x[4:5]]))


def test_silu_matches_library_and_torch():
    x = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(silu(x), x * expit(x), rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(silu(x), torch.nn.functional.silu(torch.tensor(x)).numpy(),
                               rtol=1e-14)


def test_l2_normalise_unit_norm_and_direction():
    x = R.standard_normal((50, 3, 16)) * R.uniform(0.1, 10, (50, 3, 1))
    y = l2_normalize(x)
    s = np.sum(x * x, axis=-1)
    np.testing.assert_allclose(np.sum(y * y, axis=-1), s / (s + L2_EPS), rtol=1e-13)
    cos = np.sum(x * y, axis=-1) / (np.linalg.norm(x, axis=-1) * np.linalg.norm(y, axis=-1))
    np.testing.assert_allclose(cos, 1.0, rtol=1e-14)


def test_prologue_layout_and_composition():
    """Channel p*H*D + h*D + d feeds (q, k, v)[p] at head h, channel d; q and
    k come out unit-normalised after SiLU; v is SiLU of the conv only."""
    T, H, D = 21, 3, 8
    x = R.standard_normal((T, 3 * H * D))
    w = R.standard_normal((3 * H * D, 4))
    q, k, v, _ = prologue(x, w, H, D)
    y = np.stack([lfilter(w[c, ::-1], [1.0], x[:, c]) for c in range(3 * H * D)], axis=1)
    y = (y * expit(y)).reshape(T, 3, H, D)
    np.testing.assert_allclose(v, y[:, 2], rtol=1e-12, atol=1e-13)
    for got, raw in ((q, y[:, 0]), (k, y[:, 1])):
        nrm = np.sqrt(np.sum(raw ** 2, axis=-1, keepdims=True) + L2_EPS)
        np.testing.assert_allclose(got, raw / nrm, rtol=1e-12, atol=1e-13)


def test_decode_steps_equal_prefill_of_the_same_tokens():
    """Prefill of T tokens then decode steps from its conv cache and final
    state reproduce a prefill of all the tokens."""
    N, H, D, T0, steps = 2, 2, 8, 7, 4
    C = 3 * H * D
    w = R.standard_normal((C, 4))
    xs = [R.standard_normal((T0 + steps, C)) for _ in range(N)]
    gs = [-5 * expit(R.standard_normal((T0 + steps, H, D))) for _ in range(N)]
    bs = [expit(R.standard_normal((T0 + steps, H))) for _ in range(N)]
    lengths = [T0 + steps] * N
    cu = np.concatenate([[0], np.cumsum(lengths)])
    X = np.concatenate(xs)
    q, k, v, _ = prologue(X, w, H, D, cu)
    o_full, S_full = kda_recurrent(q, k, v, np.concatenate(gs), np.concatenate(bs), 1.0, None, cu)
    # prefill of the first T0 tokens of each sequence
    cu0 = np.arange(N + 1) * T0
    X0 = np.concatenate([x[:T0] for x in xs])
    q0, k0, v0, cache = prologue(X0, w, H, D, cu0)
    _, S = kda_recurrent(q0, k0, v0, np.concatenate([g[:T0] for g in gs]),
                         np.concatenate([b[:T0] for b in bs]), 1.0, None, cu0)
    for s in range(steps):
        xt = np.stack([x[T0 + s] for x in xs])
        o, S, cache = kda_decode_step(xt, w, cache, np.stack([g[T0 + s] for g in gs]),
                                      np.stack([b[T0 + s] for b in bs]), S, H, D)
        for n in range(N):
            np.testing.assert_allclose(o[n], o_full[cu[n] + T0 + s], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S_full, rtol=1e-12, atol=1e-12)
