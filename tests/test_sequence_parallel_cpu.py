"""One sequence split across ranks, on CPU: gloo ranks stand in for GPUs and the
three steps (map of a stretch, composition, prefill of a stretch) are the
float64 oracle's, so these tests check the exchange and the order of the
composition (kda_chunk_fwd_sequence_parallel) against the whole-sequence
recurrence.  The GPU kernels behind the same steps are checked in
test_gpu_sequence_parallel.py."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import kda_recurrent, state_from_abi, state_to_abi


class OracleOps:
    """The prefill of a stretch is affine in its entry state: final = M S0 + B.
    M is the final state from the identity with v = 0 (B is linear in v and M
    depends on k, g, beta only), B the final state from a zero start; all in
    the library's layout (column-major like a state)."""

    def map(self, q, k, v, g, beta):
        T, H, D = k.shape
        eye = np.broadcast_to(np.eye(D), (1, H, D, D)).copy()
        _, Mk = kda_recurrent(q, k, np.zeros((T, H, D)), g, beta, 1.0, eye)
        _, Bk = kda_recurrent(q, k, v, g, beta, 1.0, None)
        return torch.from_numpy(state_to_abi(Mk)), torch.from_numpy(state_to_abi(Bk))

    def compose(self, M, B, E):
        Mk, Bk = state_from_abi(M.numpy()), state_from_abi(B.numpy())
        if E is None:
            return B.clone()
        Ek = state_from_abi(E.numpy())
        return torch.from_numpy(state_to_abi(np.einsum("nhik,nhkj->nhij", Mk, Ek) + Bk))

    def fwd(self, q, k, v, g, beta, o, scale, initial_state, final_state):
        s0 = None if initial_state is None else state_from_abi(initial_state.numpy())
        out, S = kda_recurrent(q, k, v, g, beta, scale, s0)
        o.copy_(torch.from_numpy(out))
        final_state.copy_(torch.from_numpy(state_to_abi(S)))


def problem(T, H, D, seed):
    r = np.random.default_rng(seed)
    q = r.standard_normal((T, H, D))
    k = r.standard_normal((T, H, D))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((T, H, D))
    g = -2.0 / (1.0 + np.exp(-r.standard_normal((T, H, D))))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((T, H))))
    s0 = 0.3 * r.standard_normal((1, H, D, D))
    return q, k, v, g, beta, s0


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, cuts, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from gated_delta_rule_prologue_b200.sequence_parallel import (
            kda_chunk_fwd_sequence_parallel)
        q, k, v, g, beta, s0 = problem(cuts[-1], 2, 6, seed=7)
        a, b = cuts[rank], cuts[rank + 1]
        sl = lambda x: torch.from_numpy(np.ascontiguousarray(x[a:b]))
        o = torch.empty((b - a, 2, 6), dtype=torch.float64)
        fs = kda_chunk_fwd_sequence_parallel(
            sl(q), sl(k), sl(v), sl(g), sl(beta), o, scale=0.5,
            initial_state=torch.from_numpy(state_to_abi(s0)), ops=OracleOps())
        out[rank] = (o.numpy().copy(), fs.numpy().copy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [[0, 9, 20], [0, 4, 5, 17]], ids=["2_ranks", "3_ranks"])
def test_split_sequence_equals_whole_sequence(cuts):
    world = len(cuts) - 1
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, cuts, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    q, k, v, g, beta, s0 = problem(cuts[-1], 2, 6, seed=7)
    o_ref, S_ref = kda_recurrent(q, k, v, g, beta, 0.5, s0)
    o = np.concatenate([out[r][0] for r in range(world)], axis=0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)
    for r in range(world):  # every rank returns the sequence's final state
        np.testing.assert_allclose(out[r][1], state_to_abi(S_ref), rtol=1e-10, atol=1e-12)


def test_single_process_runs_the_stretch_from_the_initial_state():
    from gated_delta_rule_prologue_b200.sequence_parallel import kda_chunk_fwd_sequence_parallel
    q, k, v, g, beta, s0 = problem(11, 2, 5, seed=3)
    o = torch.empty((11, 2, 5), dtype=torch.float64)
    fs = kda_chunk_fwd_sequence_parallel(*(torch.from_numpy(x) for x in (q, k, v, g, beta)), o,
                                         initial_state=torch.from_numpy(state_to_abi(s0)),
                                         ops=OracleOps())
    o_ref, S_ref = kda_recurrent(q, k, v, g, beta, 1.0, s0)
    np.testing.assert_allclose(o.numpy(), o_ref, rtol=1e-12)
    np.testing.assert_allclose(fs.numpy(), state_to_abi(S_ref), rtol=1e-12)


def test_oracle_map_is_the_affine_map_of_the_stretch():
    """final(S0) = M S0 + B for any S0: the map the ranks exchange is exact."""
    q, k, v, g, beta, s0 = problem(9, 2, 4, seed=5)
    ops = OracleOps()
    M, B = ops.map(q, k, v, g, beta)
    _, S = kda_recurrent(q, k, v, g, beta, 1.0, s0)
    E = ops.compose(M, B, torch.from_numpy(state_to_abi(s0)))
    np.testing.assert_allclose(E.numpy(), state_to_abi(S), rtol=1e-12, atol=1e-13)
