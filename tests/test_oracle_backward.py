"""Pins of the oracle's backward pass (kda_recurrent_backward).

The oracle's gradients are checked against things other than themselves:
central finite differences of the forward oracle, the calculus of the worked
example on "Kimi K3的线性注意力：从源码看懂KDA如何更新记忆" (第四站: read 10,
target 14, beta 0.5 -> 12, 13, 13.5), and closed forms for a state that
neither decays nor is written.
"""
import numpy as np
import pytest

from conftest import read_golden
from oracle import kda_recurrent, kda_recurrent_backward

RNG = np.random.default_rng(2024)


def problem(T, H, Dk, Dv, lengths=None, s0=True, seed=0):
    r = np.random.default_rng(seed)
    q = r.standard_normal((T, H, Dk))
    k = r.standard_normal((T, H, Dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((T, H, Dv))
    g = -2.0 / (1.0 + np.exp(-r.standard_normal((T, H, Dk))))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((T, H))))
    N = 1 if lengths is None else len(lengths)
    S0 = 0.5 * r.standard_normal((N, H, Dk, Dv)) if s0 else None
    cu = None if lengths is None else np.concatenate([[0], np.cumsum(lengths)])
    do = r.standard_normal((T, H, Dv))
    dSN = r.standard_normal((N, H, Dk, Dv))
    return q, k, v, g, beta, S0, cu, do, dSN


def loss(q, k, v, g, beta, S0, cu, do, dSN, scale):
    o, S = kda_recurrent(q, k, v, g, beta, scale, S0, cu)
    return float(np.sum(o * do) + np.sum(S * dSN))


@pytest.mark.parametrize("lengths", [None, [3, 0, 4]])
def test_backward_matches_central_differences(lengths):
    """Every gradient entry against (L(x + h) - L(x - h)) / 2h, h = 1e-6."""
    T, H, Dk, Dv, scale = 7, 2, 3, 2, 0.7
    q, k, v, g, beta, S0, cu, do, dSN = problem(T, H, Dk, Dv, lengths, seed=1)
    grads = kda_recurrent_backward(q, k, v, g, beta, do, dSN, scale, S0, cu)
    names = ["q", "k", "v", "g", "beta", "S0"]
    args = dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0)
    h = 1e-6
    for name, grad in zip(names, grads):
        x = args[name]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            lp = loss(cu=cu, do=do, dSN=dSN, scale=scale, **args)
            x[idx] = old - h
            lm = loss(cu=cu, do=do, dSN=dSN, scale=scale, **args)
            x[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-7, err_msg=name)


def test_backward_worked_example():
    """The first station-4 example read as a function of its inputs: with no
    decay, a unit key and q = k, the read after T writes is
    r_T = target - (target - r_0)(1 - beta)^T, so d r_T / d r_0 = (1 - beta)^T,
    d r_T / d beta_s = (target - r_{s-1})(1 - beta)^(T-s) and
    d r_T / d v_s = beta (1 - beta)^(T-s), with r_{s-1} the printed reads."""
    ex = read_golden("w1_station4_read10_target14.txt")
    reads, b, target, r0 = ex["reads"], ex["beta"], ex["target"], ex["read0"]
    T = len(reads)
    q = np.ones((T, 1, 1))
    k = np.ones((T, 1, 1))
    v = np.full((T, 1, 1), target)
    g = np.zeros((T, 1, 1))
    beta = np.full((T, 1), b)
    S0 = np.full((1, 1, 1, 1), r0)
    do = np.zeros((T, 1, 1))
    do[T - 1] = 1.0                       # loss = the last read
    dq, dk, dv, dg, dbeta, ds0 = kda_recurrent_backward(q, k, v, g, beta, do, None, 1.0, S0)
    prev = [r0] + reads[:-1]
    for s in range(T):
        np.testing.assert_allclose(dbeta[s, 0], (target - prev[s]) * (1 - b) ** (T - 1 - s),
                                   rtol=1e-14)
        np.testing.assert_allclose(dv[s, 0, 0], b * (1 - b) ** (T - 1 - s), rtol=1e-14)
    np.testing.assert_allclose(ds0[0, 0, 0, 0], (1 - b) ** T, rtol=1e-14)
    # the read is S_T q with q = 1: d/dq of the last read is the last read
    np.testing.assert_allclose(dq[T - 1, 0, 0], reads[-1], rtol=1e-14)
    # one write, loss = the state after it (through d_final_state, no read):
    # r_1 = a r_0 + b k (v - a r_0 k) with a = exp(g), so
    # d/dk = b (v - a r_0) - b a r_0 = -3 and d/dg = a r_0 (1 - b) = 5
    dq1, dk1, dv1, dg1, db1, ds1 = kda_recurrent_backward(
        q[:1], k[:1], v[:1], g[:1], beta[:1], np.zeros((1, 1, 1)), np.ones((1, 1, 1, 1)), 1.0,
        S0)
    assert dk1[0, 0, 0] == pytest.approx(b * (target - r0) - b * r0, abs=1e-14)
    assert dk1[0, 0, 0] == pytest.approx(-3.0, abs=1e-14)
    assert dg1[0, 0, 0] == pytest.approx(r0 * (1 - b), abs=1e-14)
    assert dg1[0, 0, 0] == pytest.approx(5.0, abs=1e-14)


def test_backward_closed_form_without_decay_or_write():
    """g = 0 and beta = 0: o_t = scale S0^T q_t and the final state is S0, so
    dq_t = scale S0 do_t, d S0 = scale sum_t q_t do_t^T + dSN, dv = dk = 0,
    dbeta_t = k_t^T R_t (v_t - S0^T k_t) and dg_t = rowsum(R_t * S0) with
    R_t = dSN + scale sum_{s >= t} q_s do_s^T."""
    T, H, Dk, Dv, scale = 6, 2, 4, 3, 0.5
    q, k, v, g, beta, S0, cu, do, dSN = problem(T, H, Dk, Dv, seed=3)
    g[:] = 0.0
    beta[:] = 0.0
    dq, dk, dv, dg, dbeta, ds0 = kda_recurrent_backward(q, k, v, g, beta, do, dSN, scale, S0)
    S = S0[0]
    np.testing.assert_allclose(dq, scale * np.einsum("hkv,thv->thk", S, do), rtol=1e-13)
    np.testing.assert_allclose(ds0[0], dSN[0] + scale * np.einsum("thk,thv->hkv", q, do),
                               rtol=1e-13)
    assert np.all(dv == 0) and np.all(dk == 0)
    for t in range(T):
        R = dSN[0] + scale * np.einsum("shk,shv->hkv", q[t:], do[t:])
        err = v[t] - np.einsum("hkv,hk->hv", S, k[t])
        np.testing.assert_allclose(dbeta[t], np.einsum("hk,hkv,hv->h", k[t], R, err),
                                   rtol=1e-12)
        np.testing.assert_allclose(dg[t], np.sum(R * S, axis=-1), rtol=1e-12)


@pytest.mark.parametrize("lengths,chunk", [(None, 3), ([5, 0, 9, 1], 4), ([13], 16), ([7, 6], 2)])
def test_chunkwise_backward_equals_recurrent_backward(lengths, chunk):
    """The chunk-by-chunk chain rule (second oracle) reaches the token-level
    adjoint up to rounding, for ragged chunks, empty sequences and chunk sizes
    from 2 to 16."""
    from oracle import kda_chunkwise_backward
    T = 14 if lengths is None else sum(lengths)
    q, k, v, g, beta, S0, cu, do, dSN = problem(T, 2, 4, 3, lengths, seed=5)
    ref = kda_recurrent_backward(q, k, v, g, beta, do, dSN, 0.8, S0, cu)
    got = kda_chunkwise_backward(q, k, v, g, beta, do, dSN, 0.8, S0, cu, chunk=chunk)
    for a, b in zip(ref, got):
        np.testing.assert_allclose(b, a, rtol=1e-10, atol=1e-12 * np.max(np.abs(a)))
