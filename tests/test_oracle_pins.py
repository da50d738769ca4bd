"""Pins for the float64 oracle's recurrence and chunkwise evaluator.

Each test fixes the oracle to something other than itself: a value printed on
the source pages (fixtures under tests/golden), a closed form, an invariant,
or a differently written formula from the pages.

Sources: [W1] "Kimi K3的线性注意力：从源码看懂KDA如何更新记忆";
[W3] "Kimi K3 记忆架构总览：KDA、MLA、AttnRes 各管什么";
[W5] "AI-Workshop 文献分享 #16 — KDA：给长文本建立可更新的记忆".
"""
import numpy as np
import pytest

from conftest import read_golden
from oracle import kda_chunkwise, kda_recurrent

RNG = np.random.default_rng(1234)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_problem(T, H, Dk, Dv, *, g_lo=-5.0, seed=0, s0=True, N=1):
    r = np.random.default_rng(seed)
    q = _unit(r.standard_normal((T, H, Dk)))
    k = _unit(r.standard_normal((T, H, Dk)))
    v = r.standard_normal((T, H, Dv))
    g = g_lo * (1.0 / (1.0 + np.exp(-r.standard_normal((T, H, Dk)))))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((T, H))))
    S0 = 0.3 * r.standard_normal((N, H, Dk, Dv)) if s0 else None
    return q, k, v, g, beta, S0


# --- worked examples printed on the pages ---------------------------------

def test_w1_station4_read10_target14_exact():
    """[W1 第四站]: read 10, target 14, beta 0.5 -> 12, 13, 13.5 (exact)."""
    ex = read_golden("w1_station4_read10_target14.txt")
    reads = ex["reads"]
    T, Dk, Dv = len(reads), 3, 2
    e0 = np.array([1.0, 0.0, 0.0])
    S0 = np.zeros((1, 1, Dk, Dv))
    S0[0, 0, 0] = [ex["read0"], 5.0]
    S0[0, 0, 1:] = RNG.standard_normal((Dk - 1, Dv))   # other rows: untouched
    k = np.tile(e0, (T, 1, 1))
    q = k.copy()
    v = np.tile(np.array([ex["target"], 5.0]), (T, 1, 1))
    g = np.zeros((T, 1, Dk))
    beta = np.full((T, 1), ex["beta"])
    o, S = kda_recurrent(q, k, v, g, beta, 1.0, S0)
    assert o[:, 0, 0].tolist() == reads                  # bit-exact
    assert np.all(o[:, 0, 1] == 5.0)
    assert np.array_equal(S[0, 0, 1:], S0[0, 0, 1:])
    oc, Sc = kda_chunkwise(q, k, v, g, beta, 1.0, S0, chunk=2)
    np.testing.assert_allclose(oc[:, 0, 0], reads, rtol=0, atol=1e-12)


def test_w5_s8_4_one_dim():
    """[W5 §8.4]: 0.7 with target 0.9 and beta 0.5 lands at 0.8."""
    ex = read_golden("w5_s8_4_one_dim.txt")
    one = np.ones((1, 1, 1))
    o, S = kda_recurrent(one, one, ex["target"] * one, np.zeros((1, 1, 1)),
                         np.full((1, 1), ex["beta"]), 1.0, ex["read0"] * np.ones((1, 1, 1, 1)))
    assert abs(o[0, 0, 0] - ex["reads"]) <= 2e-16
    assert abs(S[0, 0, 0, 0] - ex["reads"]) <= 2e-16


def test_w5_s5_1_orthogonal_addresses_exact():
    """[W5 §5.1]: two one-hot keys written into an empty state; querying each
    address returns its value exactly and the state's rows are the values."""
    ex = read_golden("w5_s5_1_orthogonal_keys.txt")
    kp, ko = np.array(ex["key_place"]), np.array(ex["key_occupation"])
    a = RNG.standard_normal(5)
    b = RNG.standard_normal(5)
    # tokens: write (place, a), write (occupation, b), then two pure queries
    k = np.stack([kp, ko, kp, ko])[:, None, :]
    q = np.stack([kp, ko, np.array(ex["query_place"]), np.array(ex["query_occupation"])])[:, None, :]
    v = np.stack([a, b, np.zeros(5), np.zeros(5)])[:, None, :]
    beta = np.array([[1.0], [1.0], [0.0], [0.0]])
    g = np.zeros((4, 1, 2))
    o, S = kda_recurrent(q, k, v, g, beta)
    assert np.array_equal(o[2, 0], a) and np.array_equal(o[3, 0], b)
    assert np.array_equal(S[0, 0], np.stack([a, b]))


# --- invariants and closed forms ------------------------------------------

def test_beta0_no_decay_leaves_state_unchanged():
    q, k, v, g, beta, S0 = _rand_problem(23, 3, 8, 6)
    o, S = kda_recurrent(q, k, v, np.zeros_like(g), np.zeros_like(beta), 1.0, S0)
    assert np.array_equal(S, S0)
    np.testing.assert_allclose(o, np.einsum("hkv,thk->thv", S0[0], q), rtol=1e-13, atol=1e-15)


def test_beta0_decay_closed_form():
    """beta = 0: S_T = diag(exp(sum_t g_t)) S0 and o_t = (diag(exp(sum_{j<=t} g_j)) S0)^T q_t."""
    q, k, v, g, beta, S0 = _rand_problem(40, 2, 8, 4)
    scale = 0.37
    o, S = kda_recurrent(q, k, v, g, np.zeros_like(beta), scale, S0)
    G = np.exp(np.cumsum(g, axis=0))                        # [T, H, Dk]
    np.testing.assert_allclose(S[0], G[-1][:, :, None] * S0[0], rtol=1e-12)
    ref = scale * np.einsum("thk,hkv,thk->thv", G, S0[0], q)
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-14)


def test_unit_key_beta1_writes_value_exactly():
    """Unit key, beta = 1: after the step S^T k = v, whatever the decay."""
    T, H, Dk, Dv = 12, 2, 8, 5
    q, k, v, g, beta, S0 = _rand_problem(T, H, Dk, Dv)
    beta = np.ones_like(beta)
    o, _ = kda_recurrent(k, k, v, g, beta, 1.0, S0)          # query = key
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


def test_decay_before_prediction_closed_form():
    """Same unit key every step, same decay a on every channel: the read x_t
    along the key obeys x_t = (1-beta) a x_{t-1} + beta v, so
    x_T = c^T x_0 + beta v (1 - c^T) / (1 - c) with c = (1-beta) a.
    Predicting from the undecayed state would give a different map."""
    T, Dk = 30, 4
    a, bta, vv, x0 = 0.83, 0.35, 2.5, -1.25
    e = np.zeros(Dk); e[1] = 1.0
    k = np.tile(e, (T, 1, 1)); q = k.copy()
    v = np.full((T, 1, 1), vv)
    g = np.full((T, 1, Dk), np.log(a))
    S0 = np.zeros((1, 1, Dk, 1)); S0[0, 0, 1, 0] = x0
    o, _ = kda_recurrent(q, k, v, g, np.full((T, 1), bta), 1.0, S0)
    c = (1 - bta) * a
    t = np.arange(1, T + 1)
    ref = c ** t * x0 + bta * vv * (1 - c ** t) / (1 - c)
    np.testing.assert_allclose(o[:, 0, 0], ref, rtol=1e-13)


def test_w3_reparameterised_matrix_form():
    """[W3 KDA 谱系速查]: with the value-first state M = S^T the step is
    M_t = M_{t-1}(I - beta k k^T) + beta v k^T; with per-channel decay the
    decayed state M_{t-1} diag(alpha_t) takes M_{t-1}'s place."""
    T, H, Dk, Dv = 17, 2, 6, 5
    q, k, v, g, beta, S0 = _rand_problem(T, H, Dk, Dv, seed=7)
    scale = 0.5
    o, S = kda_recurrent(q, k, v, g, beta, scale, S0)
    for h in range(H):
        M = S0[0, h].T.copy()
        for t in range(T):
            kt = k[t, h][:, None]
            M = (M @ np.diag(np.exp(g[t, h]))) @ (np.eye(Dk) - beta[t, h] * kt @ kt.T) \
                + beta[t, h] * v[t, h][:, None] @ kt.T
            np.testing.assert_allclose(o[t, h], scale * M @ q[t, h], rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(S[0, h], M.T, rtol=1e-11, atol=1e-13)


def test_w3_delta_rule_pseudocode_without_decay():
    """[W3 KDA 谱系速查] row-vector pseudocode: v_old = k @ S;
    u = beta (v - v_old); S = S + k.T @ u  (no decay)."""
    T, H, Dk, Dv = 15, 1, 7, 3
    q, k, v, g, beta, S0 = _rand_problem(T, H, Dk, Dv, seed=9)
    o, S = kda_recurrent(q, k, v, np.zeros_like(g), beta, 1.0, S0)
    Sp = S0[0, 0].copy()
    for t in range(T):
        kr = k[t, 0][None, :]
        v_old = kr @ Sp
        u = beta[t, 0] * (v[t, 0][None, :] - v_old)
        Sp = Sp + kr.T @ u
        np.testing.assert_allclose(o[t, 0], (q[t, 0][None, :] @ Sp)[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S[0, 0], Sp, rtol=1e-12, atol=1e-13)


def test_value_rotation_equivariance():
    """Rotating the value space (V R, S0 R) rotates outputs and final state."""
    q, k, v, g, beta, S0 = _rand_problem(20, 2, 6, 5, seed=3)
    R, _ = np.linalg.qr(RNG.standard_normal((5, 5)))
    o, S = kda_recurrent(q, k, v, g, beta, 1.0, S0)
    o2, S2 = kda_recurrent(q, k, v @ R, g, beta, 1.0, S0 @ R)
    np.testing.assert_allclose(o2, o @ R, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S2, S @ R, rtol=1e-11, atol=1e-12)


def test_key_channel_permutation_invariance():
    """Permuting key channels of q, k, g and the state's rows changes nothing
    but the order of the final state's rows (decay is per key channel)."""
    q, k, v, g, beta, S0 = _rand_problem(20, 2, 6, 5, seed=4)
    p = RNG.permutation(6)
    o, S = kda_recurrent(q, k, v, g, beta, 1.0, S0)
    o2, S2 = kda_recurrent(q[..., p], k[..., p], v, g[..., p], beta, 1.0, S0[:, :, p, :])
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S2, S[:, :, p, :], rtol=1e-12, atol=1e-13)


def test_joint_linearity_in_values_and_state():
    q, k, v, g, beta, S0 = _rand_problem(18, 2, 6, 4, seed=5)
    _, _, v2, _, _, S02 = _rand_problem(18, 2, 6, 4, seed=6)
    a, b = 0.7, -1.9
    o1, F1 = kda_recurrent(q, k, v, g, beta, 1.0, S0)
    o2, F2 = kda_recurrent(q, k, v2, g, beta, 1.0, S02)
    o3, F3 = kda_recurrent(q, k, a * v + b * v2, g, beta, 1.0, a * S0 + b * S02)
    np.testing.assert_allclose(o3, a * o1 + b * o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(F3, a * F1 + b * F2, rtol=1e-11, atol=1e-12)


def test_varlen_equals_separate_runs():
    lengths = [5, 1, 17, 9]
    T = sum(lengths)
    q, k, v, g, beta, S0 = _rand_problem(T, 2, 6, 4, seed=8, N=len(lengths))
    cu = np.concatenate([[0], np.cumsum(lengths)])
    o, S = kda_recurrent(q, k, v, g, beta, 1.0, S0, cu)
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        on, Sn = kda_recurrent(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], 1.0, S0[n:n + 1])
        assert np.array_equal(o[a:b], on) and np.array_equal(S[n], Sn[0])


def test_resume_from_final_state_equals_one_pass():
    q, k, v, g, beta, S0 = _rand_problem(30, 2, 6, 4, seed=10)
    o, S = kda_recurrent(q, k, v, g, beta, 1.0, S0)
    o1, S1 = kda_recurrent(q[:13], k[:13], v[:13], g[:13], beta[:13], 1.0, S0)
    o2, S2 = kda_recurrent(q[13:], k[13:], v[13:], g[13:], beta[13:], 1.0, S1)
    np.testing.assert_array_equal(np.concatenate([o1, o2]), o)
    np.testing.assert_array_equal(S2, S)


# --- chunkwise evaluator against the recurrence -----------------------------

@pytest.mark.parametrize("chunk", [1, 2, 4, 16, 64])
def test_chunkwise_equals_recurrence(chunk):
    lengths = [50, 3, 77]                  # ragged tails, a sequence shorter than a chunk
    T = sum(lengths)
    q, k, v, g, beta, S0 = _rand_problem(T, 2, 8, 6, seed=11, N=len(lengths))
    cu = np.concatenate([[0], np.cumsum(lengths)])
    o, S = kda_recurrent(q, k, v, g, beta, 0.8, S0, cu)
    oc, Sc = kda_chunkwise(q, k, v, g, beta, 0.8, S0, cu, chunk=chunk)
    assert np.max(np.abs(oc - o)) <= 1e-12 * np.sqrt(np.mean(o * o))
    assert np.linalg.norm(Sc - S) <= 1e-12 * np.linalg.norm(S)


def test_chunkwise_slow_decay_and_saturated_decay():
    for g_lo in (-0.06, -5.0):
        q, k, v, g, beta, S0 = _rand_problem(130, 1, 16, 16, g_lo=g_lo, seed=12)
        if g_lo == -5.0:
            g = np.full_like(g, -5.0)      # cumulative -320 over a 64-token chunk
        o, S = kda_recurrent(q, k, v, g, beta, 1.0, S0)
        oc, Sc = kda_chunkwise(q, k, v, g, beta, 1.0, S0, chunk=64)
        assert np.all(np.isfinite(oc))
        assert np.max(np.abs(oc - o)) <= 1e-11 * np.sqrt(np.mean(o * o))
        assert np.linalg.norm(Sc - S) <= 1e-11 * max(np.linalg.norm(S), 1e-300)
