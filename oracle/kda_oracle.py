"""Float64 CPU oracle for the Kimi Delta Attention (KDA) recurrence hot path.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
baseline may import this module.  It is deliberately plain and slow: NumPy in
float64, a Python loop over tokens, no blocking or fusion beyond what each
definition states.  It shares no code with the CUDA path.

Sources (web pages; cited as [Wn section]):

  [W1] "Kimi K3的线性注意力：从源码看懂KDA如何更新记忆" (yeyulingfeng.com) --
       the stations 第二站 (short conv, SiLU, L2), 第三站 (per-channel decay),
       第四站 (delta-rule write; naive_recurrent_kda excerpt), 第五站 (read
       after write; query scale), 第六站 (per-head RMSNorm and output gate),
       彩蛋 (chunked execution; bounded gate, the gate.py excerpt).
  [W3] "Kimi K3 记忆架构总览：KDA、MLA、AttnRes 各管什么" (moonzj.com),
       section "KDA 谱系速查" (delta-rule pseudocode, reparameterisation).
  [W4] "KimiK3轻量化复刻实现KDA并行解析，Chunkwise并行与状态压缩机制详解"
       (tech.news18a.com) -- ShortConv paragraph (width 4, current token and
       three previous ones, per channel) and Figure 1 (affine chunk map).
  [W5] "AI-Workshop 文献分享 #16 — KDA：给长文本建立可更新的记忆" --
       §5.1, §8.4, §10.3.

Readings where the pages are silent or garbled (each one is listed in the
repository's design notes):

  * Order inside a token: decay, then predict from the decayed state, then
    write, then read ([W1 第三站/第四站/第五站]; the excerpt of
    naive_recurrent_kda applies ``S * exp(g)`` before the error term).  [W5
    §8.3]'s simplified form that predicts from the undecayed state is not used.
  * State is key-first, ``S[Dk, Dv]`` ([W1 第三站]).  Inputs/outputs in the
    ABI's ``[N, H, Dv, Dk]`` layout are transposed by the caller of this
    module.
  * Query scale: a plain multiplier on the read ([W1 第五站] leaves its value
    open); default 1.
  * Short conv ([W1 第二站], [W4 ShortConv]): depthwise, width 4, no bias;
    tap 3 multiplies the current token and tap 0 the token three back;
    history before a sequence start is the given cache (oldest row first) or
    zero; the conv never crosses a ``cu_seqlens`` boundary.  SiLU(x) =
    x*sigmoid(x) follows the conv on q, k and v.
  * L2 normalisation of q and k per (token, head) over the head's channels:
    ``x / sqrt(sum(x^2) + 1e-6)`` (the epsilon is ours).
"""
from __future__ import annotations

import numpy as np

L2_EPS = 1e-6


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor (any dtype, incl. bfloat16)
        a = a.detach().cpu()
        if str(a.dtype) == "torch.bfloat16":
            a = a.float()
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


def _segments(T, cu_seqlens):
    if cu_seqlens is None:
        return [(0, T)]
    cu = [int(c) for c in np.asarray(_f64(cu_seqlens)).astype(np.int64)]
    return list(zip(cu[:-1], cu[1:]))


# ---------------------------------------------------------------------------
# Prologue: causal depthwise short conv, SiLU, L2 normalisation
# ---------------------------------------------------------------------------

def silu(x):
    """SiLU(x) = x * sigmoid(x) ([W1 第二站]: activation inside the short conv)."""
    return x / (1.0 + np.exp(-x))


def short_conv(x, w, cu_seqlens=None, cache_in=None):
    """Causal depthwise conv of width 4 over packed tokens, no activation.

    ``x`` [T, C]; ``w`` [C, 4]; ``cache_in`` [N, 3, C] (oldest first) or None.
    Returns ``(y [T, C], cache_out [N, 3, C])`` where
    ``y[t, c] = sum_j w[c, j] * x[t - 3 + j, c]`` with positions before the
    sequence start taken from the cache (or zero), and ``cache_out[n]`` holds
    the last three inputs of sequence n (cache rows if the sequence is
    shorter than three).  [W1 第二站]; [W4 ShortConv paragraph].
    """
    x = _f64(x)
    w = _f64(w)
    T, C = x.shape
    segs = _segments(T, cu_seqlens)
    y = np.zeros((T, C))
    cache_out = np.zeros((len(segs), 3, C))
    for n, (a, b) in enumerate(segs):
        hist = np.zeros((3, C)) if cache_in is None else _f64(cache_in)[n]
        ext = np.concatenate([hist, x[a:b]], axis=0)      # ext[i] is token a-3+i
        for t in range(b - a):
            window = ext[t:t + 4]                          # tokens t-3 .. t
            y[a + t] = np.einsum("jc,cj->c", window, w)
        cache_out[n] = ext[-3:]
    return y, cache_out


def l2_normalize(x, eps=L2_EPS):
    """Per-row unit normalisation ``x / sqrt(sum x^2 + eps)`` over the last axis."""
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def prologue(x, w, H, D, cu_seqlens=None, cache_in=None):
    """Short conv + SiLU on the q/k/v projections, then L2 on q and k.

    ``x`` [T, 3*H*D] with channel ``p*H*D + h*D + d`` (p: 0 query, 1 key,
    2 value).  Returns ``q, k, v`` [T, H, D] float64 and the new conv cache.
    [W1 第二站]: conv and SiLU first; q and k are normalised afterwards.
    """
    y, cache_out = short_conv(x, w, cu_seqlens, cache_in)
    y = silu(y)
    T = y.shape[0]
    y = y.reshape(T, 3, H, D)
    q = l2_normalize(y[:, 0])
    k = l2_normalize(y[:, 1])
    v = y[:, 2].copy()
    return q, k, v, cache_out


# ---------------------------------------------------------------------------
# The recurrence (definition)
# ---------------------------------------------------------------------------

def gate(g_raw, A_log=None, dt_bias=None, lower_bound=-5.0):
    """Bounded log-decay from the gate pre-activations ([W1 彩蛋], the excerpt of
    FLA's gate.py): add the per-(head, channel) bias, multiply by exp(A_log) of
    the head, squash with a sigmoid and scale by the lower bound (-5 in K3):

        g = lower_bound * sigmoid(exp(A_log[h]) * (g_raw + dt_bias[h, :]))

    so g lies in (lower_bound, 0) and alpha = exp(g) in (exp(lower_bound), 1).
    Either parameter may be None (the excerpt skips it then).

    g_raw [..., H, D]; A_log [H]; dt_bias [H, D].  Returns float64 g of g_raw's
    shape.
    """
    z = _f64(g_raw)
    if dt_bias is not None:
        z = z + _f64(dt_bias)
    if A_log is not None:
        z = np.exp(_f64(A_log))[:, None] * z
    # sigmoid in the form that never overflows: exp of a non-positive number only
    e = np.exp(-np.abs(z))
    sig = np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return float(lower_bound) * sig


def output_epilogue(o, gate_preact, weight, eps=1e-5):
    """Output path after the read ([W1 第六站]): per-head RMSNorm of the read-out,
    then the output gate scales each channel.  Reading of the garbled formula:
    the gate is a sigmoid of its pre-activation (a per-channel proportion in
    (0, 1)), the norm's epsilon is a parameter:

        out = o / sqrt(mean_d(o^2) + eps) * weight * sigmoid(gate_preact)

    o, gate_preact [..., D]; weight [D] (shared by the heads).  float64.
    """
    o = _f64(o)
    z = _f64(gate_preact)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + float(eps))
    e = np.exp(-np.abs(z))
    sig = np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return o / rms * _f64(weight) * sig


def kda_recurrent(q, k, v, g, beta, scale=1.0, initial_state=None, cu_seqlens=None):
    """Token-by-token KDA recurrence, all heads at once.

    Per head with key-first state ``S[Dk, Dv]`` and each token t in order:

        S   <- diag(exp(g_t)) S                 decay rows   [W1 第三站]
        e   <- v_t - S^T k_t                    prediction error [W1 第四站]
        S   <- S + beta_t k_t e^T               delta write  [W1 第四站]
        o_t <- scale * S^T q_t                  read after write [W1 第五站]

    Shapes: q, k, g [T, H, Dk]; v [T, H, Dv]; beta [T, H];
    ``initial_state`` [N, H, Dk, Dv] (key-first) or None (zeros).  The state
    restarts from ``initial_state[n]`` at each sequence start.
    Returns ``o`` [T, H, Dv] and ``final_state`` [N, H, Dk, Dv].
    """
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    T, H, Dk = k.shape
    Dv = v.shape[2]
    segs = _segments(T, cu_seqlens)
    s0 = None if initial_state is None else _f64(initial_state)
    o = np.zeros((T, H, Dv))
    final = np.zeros((len(segs), H, Dk, Dv))
    for n, (a, b) in enumerate(segs):
        S = np.zeros((H, Dk, Dv)) if s0 is None else s0[n].copy()
        for t in range(a, b):
            S = S * np.exp(g[t])[:, :, None]
            pred = np.einsum("hkv,hk->hv", S, k[t])
            err = v[t] - pred
            S = S + beta[t][:, None, None] * k[t][:, :, None] * err[:, None, :]
            o[t] = scale * np.einsum("hkv,hk->hv", S, q[t])
        final[n] = S
    return o, final


def kda_recurrent_backward(q, k, v, g, beta, do, d_final_state=None, scale=1.0,
                           initial_state=None, cu_seqlens=None):
    """Gradients of the token-by-token recurrence (reverse-mode, float64).

    The loss is taken as L = sum(do * o) + sum(d_final_state * final_state),
    with ``o`` and ``final_state`` those of :func:`kda_recurrent`; this is the
    adjoint of each step of that recurrence, taken in reverse token order:

        after the read  o_t = scale S_t^T q_t:
            dS_t += scale q_t do_t^T;          dq_t = scale S_t do_t
        after the write S_t = Sd + beta_t k_t e^T (Sd the decayed state):
            dbeta_t = k_t^T dS_t e;            dk_t = beta_t dS_t e
            de = beta_t dS_t^T k_t;            dSd = dS_t
        after the error e = v_t - Sd^T k_t:
            dv_t = de;  dSd -= k_t de^T;       dk_t -= Sd de
        after the decay Sd = diag(exp(g_t)) S_{t-1}:
            dg_t = rowsum(dSd * Sd);           dS_{t-1} = diag(exp(g_t)) dSd

    Training is mentioned on [W1 彩蛋]; the pages give no backward, so this
    is the plain chain rule through the forward definition.  Shapes as in
    :func:`kda_recurrent`; ``do`` [T, H, Dv]; ``d_final_state`` [N, H, Dk,
    Dv] (key-first) or None.  Returns dq, dk, dg [T, H, Dk], dv [T, H, Dv],
    dbeta [T, H] and d_initial_state [N, H, Dk, Dv].
    """
    q, k, v, g, beta, do = (_f64(a) for a in (q, k, v, g, beta, do))
    T, H, Dk = k.shape
    Dv = v.shape[2]
    segs = _segments(T, cu_seqlens)
    s0 = None if initial_state is None else _f64(initial_state)
    dsN = None if d_final_state is None else _f64(d_final_state)
    dq, dk, dg = np.zeros((T, H, Dk)), np.zeros((T, H, Dk)), np.zeros((T, H, Dk))
    dv, dbeta = np.zeros((T, H, Dv)), np.zeros((T, H))
    ds0 = np.zeros((len(segs), H, Dk, Dv))
    for n, (a, b) in enumerate(segs):
        # forward, keeping the decayed state, the error and the state after each token
        S = np.zeros((H, Dk, Dv)) if s0 is None else s0[n].copy()
        Sd_hist, err_hist, S_hist = [], [], []
        for t in range(a, b):
            Sd = S * np.exp(g[t])[:, :, None]
            err = v[t] - np.einsum("hkv,hk->hv", Sd, k[t])
            S = Sd + beta[t][:, None, None] * k[t][:, :, None] * err[:, None, :]
            Sd_hist.append(Sd)
            err_hist.append(err)
            S_hist.append(S)
        dS = np.zeros((H, Dk, Dv)) if dsN is None else dsN[n].copy()
        for t in range(b - 1, a - 1, -1):
            i = t - a
            Sd, err, St = Sd_hist[i], err_hist[i], S_hist[i]
            dS = dS + scale * q[t][:, :, None] * do[t][:, None, :]
            dq[t] = scale * np.einsum("hkv,hv->hk", St, do[t])
            dSe = np.einsum("hkv,hv->hk", dS, err)           # dS_t e
            dbeta[t] = np.einsum("hk,hk->h", k[t], dSe)
            de = beta[t][:, None] * np.einsum("hkv,hk->hv", dS, k[t])
            dv[t] = de
            dk[t] = beta[t][:, None] * dSe - np.einsum("hkv,hv->hk", Sd, de)
            dSd = dS - k[t][:, :, None] * de[:, None, :]
            dg[t] = np.einsum("hkv,hkv->hk", dSd, Sd)
            dS = dSd * np.exp(g[t])[:, :, None]
        ds0[n] = dS
    return dq, dk, dv, dg, dbeta, ds0


# ---------------------------------------------------------------------------
# Chunkwise evaluation (second oracle)
# ---------------------------------------------------------------------------

def _solve_unit_lower(L, rhs):
    """Solve ``L X = rhs`` for unit-lower-triangular ``L`` by forward
    substitution (row by row, in order)."""
    n = L.shape[0]
    X = np.zeros_like(rhs)
    for r in range(n):
        X[r] = rhs[r] - L[r, :r] @ X[:r]
    return X


def kda_chunkwise(q, k, v, g, beta, scale=1.0, initial_state=None, cu_seqlens=None,
                  chunk=64):
    """Chunkwise evaluation of the same recurrence, float64.

    [W1 彩蛋] and [W5 §10.3]: tokens are grouped into chunks; the state is
    passed from chunk to chunk and the work inside a chunk is matrix algebra.
    [W4 Figure 1]: a chunk maps its entry state affinely to its exit state.
    Derivation (from the recurrence; inclusive in-chunk cumulative log-decay
    ``gamma_r = sum_{j<=r} g_j``, ``G_r = exp(gamma_r)``, entry state S0):

        u_r := beta_r (v_r - (diag(alpha_r) S_{r-1})^T k_r)  gives
        S_r  = diag(G_r) S0 + sum_{i<=r} diag(G_r / G_i) k_i u_i^T.
        A[r,i] = beta_r <k_r*G_r, k_i/G_i>        for i < r  (else 0)
        (I + A) U = diag(beta) V - diag(beta) (K*G) S0
                  => U = Ut - W S0 with (I+A)[Ut | W] = [diag(beta)V | diag(beta)(K*G)]
        P[r,i] = <q_r*G_r, k_i/G_i>               for i <= r (else 0)
        O      = scale * ((Q*G) S0 + P U)
        S_exit = diag(G_last) S0 + (K * G_last / G)^T U

    The unit-lower-triangular system is solved by forward substitution.
    Same shapes and return values as :func:`kda_recurrent`.
    """
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    T, H, Dk = k.shape
    Dv = v.shape[2]
    segs = _segments(T, cu_seqlens)
    s0 = None if initial_state is None else _f64(initial_state)
    o = np.zeros((T, H, Dv))
    final = np.zeros((len(segs), H, Dk, Dv))
    for n, (a, b) in enumerate(segs):
        S = np.zeros((H, Dk, Dv)) if s0 is None else s0[n].copy()
        for c0 in range(a, b, chunk):
            c1 = min(c0 + chunk, b)
            L = c1 - c0
            for h in range(H):
                Kc, Qc, Vc = k[c0:c1, h], q[c0:c1, h], v[c0:c1, h]
                bc = beta[c0:c1, h]
                gam = np.cumsum(g[c0:c1, h], axis=0)
                G = np.exp(gam)
                KG, Kinv, QG = Kc * G, Kc / G, Qc * G
                A = np.tril(bc[:, None] * (KG @ Kinv.T), k=-1)
                P = np.tril(QG @ Kinv.T, k=0)
                rhs = np.concatenate([bc[:, None] * Vc, bc[:, None] * KG], axis=1)
                X = _solve_unit_lower(np.eye(L) + A, rhs)
                Ut, W = X[:, :Dv], X[:, Dv:]
                U = Ut - W @ S[h]
                o[c0:c1, h] = scale * (QG @ S[h] + P @ U)
                S[h] = G[-1][:, None] * S[h] + (Kc * (G[-1] / G)).T @ U
        final[n] = S
    return o, final


def _solve_unit_upper_transposed(L, rhs):
    """Solve ``L^T X = rhs`` for unit-lower-triangular ``L`` by back
    substitution (row by row, last first)."""
    n = L.shape[0]
    X = np.zeros_like(rhs)
    for r in range(n - 1, -1, -1):
        X[r] = rhs[r] - L[r + 1:, r] @ X[r + 1:]
    return X


def kda_chunkwise_backward(q, k, v, g, beta, do, d_final_state=None, scale=1.0,
                           initial_state=None, cu_seqlens=None, chunk=64):
    """Gradients of :func:`kda_chunkwise`, chunk by chunk (second oracle).

    The chain rule through the chunk algebra of :func:`kda_chunkwise`, in
    float64, with the entry state of every chunk from a forward sweep and
    the adjoint of its exit state dS' from the chunk after it (reverse sweep).
    With R = diag(beta)(V - (K*G) S0) (so U = (I + A)^{-1} R), K' = K*G_last/G
    and dO' = scale dO, per chunk:

        dU  = P^T dO' + K' dS'               dP  = lower(dO' U^T)
        dR  = (I + A)^{-T} dU                dA  = -strict_lower(dR U^T)
        dV  = diag(beta) dR                  dK' = U dS'^T
        dQG = dO' S0^T + dP (K/G)
        dKG = -diag(beta) dR S0^T + diag(beta) dA (K/G)
        dKD = (diag(beta) dA)^T (K*G) + dP^T (Q*G)
        dbeta_r = <dR_r, V_r - ((K*G) S0)_r> + sum_i dA[r,i] ((K*G)(K/G)^T)[r,i]
        dS0 = diag(G_last) dS' + (Q*G)^T dO' - (diag(beta) K*G)^T dR
        dq = dQG*G;   dk = dKG*G + dKD/G + dK'*G_last/G
        dgamma = dQG*(Q*G) + dKG*(K*G) - dKD*(K/G) - dK'*K', and on the last
                 row also + G_last*rowsum(S0*dS') + sum_i dK'_i*K'_i
        dg = reverse cumulative sum of dgamma over the chunk's rows

    (the gradient of gamma_r = sum_{j<=r} g_j).  Must agree with
    :func:`kda_recurrent_backward` up to rounding; same shapes and returns.
    """
    q, k, v, g, beta, do = (_f64(a) for a in (q, k, v, g, beta, do))
    T, H, Dk = k.shape
    Dv = v.shape[2]
    segs = _segments(T, cu_seqlens)
    s0 = None if initial_state is None else _f64(initial_state)
    dsN = None if d_final_state is None else _f64(d_final_state)
    dq, dk, dg = np.zeros((T, H, Dk)), np.zeros((T, H, Dk)), np.zeros((T, H, Dk))
    dv, dbeta = np.zeros((T, H, Dv)), np.zeros((T, H))
    ds0 = np.zeros((len(segs), H, Dk, Dv))
    for n, (a, b) in enumerate(segs):
        starts = list(range(a, b, chunk))
        # forward sweep: entry state of every chunk
        S = np.zeros((H, Dk, Dv)) if s0 is None else s0[n].copy()
        entry = []
        for c0 in starts:
            entry.append(S.copy())
            c1 = min(c0 + chunk, b)
            for h in range(H):
                Kc, Vc, bc = k[c0:c1, h], v[c0:c1, h], beta[c0:c1, h]
                G = np.exp(np.cumsum(g[c0:c1, h], axis=0))
                KG, KD = Kc * G, Kc / G
                A = np.tril(bc[:, None] * (KG @ KD.T), k=-1)
                R = bc[:, None] * (Vc - KG @ S[h])
                U = _solve_unit_lower(np.eye(c1 - c0) + A, R)
                S[h] = G[-1][:, None] * S[h] + (Kc * (G[-1] / G)).T @ U
        # reverse sweep
        dS = np.zeros((H, Dk, Dv)) if dsN is None else dsN[n].copy()
        for ci in range(len(starts) - 1, -1, -1):
            c0 = starts[ci]
            c1 = min(c0 + chunk, b)
            L = c1 - c0
            for h in range(H):
                S0c = entry[ci][h]
                Kc, Qc, Vc = k[c0:c1, h], q[c0:c1, h], v[c0:c1, h]
                bc = beta[c0:c1, h]
                G = np.exp(np.cumsum(g[c0:c1, h], axis=0))
                KG, KD, QG = Kc * G, Kc / G, Qc * G
                KK = KG @ KD.T
                A = np.tril(bc[:, None] * KK, k=-1)
                P = np.tril(QG @ KD.T, k=0)
                E = Vc - KG @ S0c
                R = bc[:, None] * E
                U = _solve_unit_lower(np.eye(L) + A, R)
                Kp = Kc * (G[-1] / G)
                dOp = scale * do[c0:c1, h]
                dSp = dS[h]
                dU = P.T @ dOp + Kp @ dSp
                dP = np.tril(dOp @ U.T, k=0)
                dR = _solve_unit_upper_transposed(np.eye(L) + A, dU)
                dA = -np.tril(dR @ U.T, k=-1)
                dKp = U @ dSp.T
                dQG = dOp @ S0c.T + dP @ KD
                dKG = -bc[:, None] * (dR @ S0c.T) + bc[:, None] * (dA @ KD)
                dKD = (bc[:, None] * dA).T @ KG + dP.T @ QG
                dv[c0:c1, h] = bc[:, None] * dR
                dbeta[c0:c1, h] = np.sum(dR * E, axis=1) + np.sum(dA * KK, axis=1)
                dq[c0:c1, h] = dQG * G
                dk[c0:c1, h] = dKG * G + dKD / G + dKp * (G[-1] / G)
                dgam = dQG * QG + dKG * KG - dKD * KD - dKp * Kp
                dgam[-1] += G[-1] * np.sum(S0c * dSp, axis=1) + np.sum(dKp * Kp, axis=0)
                dg[c0:c1, h] = np.cumsum(dgam[::-1], axis=0)[::-1]
                dS[h] = G[-1][:, None] * dSp + QG.T @ dOp - (bc[:, None] * KG).T @ dR
        ds0[n] = dS
    return dq, dk, dv, dg, dbeta, ds0


# ---------------------------------------------------------------------------
# One decode step: prologue on one new token with cache, then one update
# ---------------------------------------------------------------------------

def kda_decode_step(x, w, conv_cache, g, beta, state, H, D, scale=1.0):
    """One token per sequence for N independent sequences.

    ``x`` [N, 3*H*D]; ``conv_cache`` [N, 3, 3*H*D] (oldest first);
    ``g`` [N, H, D]; ``beta`` [N, H]; ``state`` [N, H, Dk, Dv] key-first.
    Returns ``(o [N, H, Dv], new_state, new_cache)``.  The step is the
    prologue of [W1 第二站] on a one-token sequence with the cache as history,
    followed by one application of the recurrence of :func:`kda_recurrent`
    (the recurrent mode used for generation, [W1 彩蛋]).
    """
    x = _f64(x)
    N = x.shape[0]
    cu = np.arange(N + 1)
    q, k, v, new_cache = prologue(x, w, H, D, cu_seqlens=cu, cache_in=conv_cache)
    o, new_state = kda_recurrent(q, k, v, g, beta, scale, initial_state=state,
                                 cu_seqlens=cu)
    return o, new_state, new_cache


def state_to_abi(S):
    """Key-first ``[..., Dk, Dv]`` -> the ABI's ``[..., Dv, Dk]``."""
    return np.swapaxes(_f64(S), -1, -2)


def state_from_abi(S):
    """The ABI's ``[..., Dv, Dk]`` -> key-first ``[..., Dk, Dv]``."""
    return np.swapaxes(_f64(S), -1, -2)
