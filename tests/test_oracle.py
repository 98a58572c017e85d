"""CPU tests: the fp64 oracle against what the pages and mathematics fix.

P1-P5 are closed forms / special cases of the update rule (tests/pins.py).
P6: the token recurrence and the chunkwise reformulation agree by brute force
    for many chunk sizes, ragged tails included (two independent formulations).
P7: state passing: one call over [0,T) equals two calls chained through S_T.
P8: T chained single-token decode steps equal the prefill recurrence.
P9: the chunkwise intermediate T is the inverse of (I + A).
P10-P13: the variants (delta rule, scalar gated delta rule, gated linear
    attention, plain linear attention) against their rules written out.
Mutation test: each planted mistake in the oracle makes at least one pin fail.
"""
import numpy as np
import pytest

import oracle
from tests import pins

TOL = 1e-12


def rec(mutation=None):
    return lambda q, k, v, la, b, S0: oracle.recurrent(q, k, v, la, b, S0, mutation=mutation)


def chk(C, mutation=None):
    return lambda q, k, v, la, b, S0: oracle.chunkwise(q, k, v, la, b, S0, C=C, mutation=mutation)


RUNNERS = {"recurrent": rec(), "chunkwise_c1": chk(1), "chunkwise_c4": chk(4), "chunkwise_c16": chk(16),
           "chunkwise_c64": chk(64)}


@pytest.mark.parametrize("runner", list(RUNNERS))
@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pins(pin, runner):
    assert pin(RUNNERS[runner]) < TOL


@pytest.mark.parametrize("C", [1, 2, 3, 4, 5, 8, 16, 64])
@pytest.mark.parametrize("T", [1, 7, 33, 64, 100])
def test_p6_recurrence_equals_chunkwise(C, T):
    q, k, v, la, beta, S0 = pins.random_inputs(100 + T + 7 * C, T=T, dk=6, dv=5)
    o1, s1 = oracle.recurrent(q, k, v, la, beta, S0)
    o2, s2 = oracle.chunkwise(q, k, v, la, beta, S0, C=C)
    scale = max(1.0, np.abs(o1).max())
    assert np.abs(o1 - o2).max() / scale < 1e-12
    assert np.abs(s1 - s2).max() / max(1.0, np.abs(s1).max()) < 1e-12


def test_p6_strong_decay_chunkwise():
    # Per-token decay up to e^-5: inside a 64-token chunk G reaches about -300,
    # where the printed K/Gamma form would overflow; the oracle's exponent is
    # always G_r - G_s <= 0.
    q, k, v, la, beta, S0 = pins.random_inputs(7, T=130, dk=6, dv=4, la_range=(0.5, 5.0))
    o1, s1 = oracle.recurrent(q, k, v, la, beta, S0)
    o2, s2 = oracle.chunkwise(q, k, v, la, beta, S0, C=64)
    assert np.isfinite(o2).all() and np.isfinite(s2).all()
    assert np.abs(o1 - o2).max() < 1e-12 and np.abs(s1 - s2).max() < 1e-12


@pytest.mark.parametrize("T1", [0, 1, 31, 64, 65])
def test_p7_state_passing(T1):
    q, k, v, la, beta, S0 = pins.random_inputs(21, T=97, dk=8, dv=8)
    o, ST = oracle.recurrent(q, k, v, la, beta, S0)
    oa, Sa = oracle.chunkwise(q[:, :T1], k[:, :T1], v[:, :T1], la[:, :T1], beta[:, :T1], S0, C=16)
    ob, Sb = oracle.chunkwise(q[:, T1:], k[:, T1:], v[:, T1:], la[:, T1:], beta[:, T1:], Sa, C=16)
    assert np.abs(np.concatenate([oa, ob], axis=1) - o).max() < 1e-12
    assert np.abs(Sb - ST).max() < 1e-12


def test_p8_decode_chain_equals_recurrence():
    q, k, v, la, beta, S0 = pins.random_inputs(22, T=40, dk=8, dv=6, B_=3, H_=2)
    o, ST = oracle.recurrent(q, k, v, la, beta, S0)
    S = S0
    for t in range(q.shape[1]):
        ot, S = oracle.decode_step(q[:, t], k[:, t], v[:, t], la[:, t], beta[:, t], S)
        assert np.abs(ot - o[:, t]).max() < 1e-12
    assert np.abs(S - ST).max() < 1e-12


@pytest.mark.parametrize("C", [4, 16, 64])
def test_p9_inverse(C):
    q, k, v, la, beta, S0 = pins.random_inputs(23, T=100, dk=8, dv=8)
    _, _, A, Ti = oracle.chunkwise(q, k, v, la, beta, S0, C=C, debug=True)
    eye = np.eye(C)
    res = np.einsum("bhnrs,bhnsj->bhnrj", eye + A, Ti) - eye
    assert np.abs(res).max() < 1e-12
    # A strictly lower, T unit lower triangular
    assert np.abs(np.triu(A)).max() == 0.0
    assert np.allclose(np.diagonal(Ti, axis1=-2, axis2=-1), 1.0)


def test_zero_length_and_empty_batch():
    q, k, v, la, beta, S0 = pins.random_inputs(24, T=5, dk=4, dv=4)
    o, ST = oracle.recurrent(q[:, :0], k[:, :0], v[:, :0], la[:, :0], beta[:, :0], S0)
    assert o.shape == (1, 0, 2, 4) and np.array_equal(ST, S0)
    o, ST = oracle.chunkwise(q[:, :0], k[:, :0], v[:, :0], la[:, :0], beta[:, :0], S0, C=4)
    assert np.array_equal(ST, S0)


RECURRENT_MUTANTS = ["no_decay", "decay_after", "erase_sign", "read_before", "transposed_read",
                     "beta_write_only", "decay_columns"]
CHUNKWISE_MUTANTS = ["prefix_decay_k", "strict_tril_o"]


@pytest.mark.parametrize("mutant", RECURRENT_MUTANTS + CHUNKWISE_MUTANTS)
def test_planted_mistake_is_caught(mutant):
    run = rec(mutant) if mutant in RECURRENT_MUTANTS else chk(4, mutant)
    errs = {p.__name__: p(run) for p in pins.ALL_PINS}
    # the chunkwise-only mistakes are also visible to the brute-force pin P6
    if mutant in CHUNKWISE_MUTANTS:
        q, k, v, la, beta, S0 = pins.random_inputs(31, T=20, dk=8, dv=8)
        o1, s1 = oracle.recurrent(q, k, v, la, beta, S0)
        o2, s2 = run(q, k, v, la, beta, S0)
        errs["p6"] = max(np.abs(o1 - o2).max(), np.abs(s1 - s2).max())
    assert max(errs.values()) > 1e-6, errs


def test_hand_worked_example():
    """Two tokens worked by hand from the update rule (tests/golden)."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked_t2_d2.json")))
    q = np.array(g["q"])[None, :, None]
    k = np.array(g["k"])[None, :, None]
    v = np.array(g["v"])[None, :, None]
    la = np.log(np.array(g["alpha"]))[None, :, None]
    beta = np.array(g["beta"])[None, :, None]
    S0 = np.array(g["S0"])[None, None]
    for run in (rec(), chk(1), chk(2), chk(64)):
        o, ST = run(q, k, v, la, beta, S0)
        assert np.abs(o[0, :, 0] - np.array(g["o"])).max() < 1e-12
        assert np.abs(ST[0, 0] - np.array(g["S_T"])).max() < 1e-12


# ---------------------------------------------------------------- variants


def vrec(mutation=None):
    return lambda q, k, v, la, b, S0, erase, gate: oracle.recurrent(q, k, v, la, b, S0, mutation=mutation,
                                                                   erase=erase, gate=gate)


def vchk(C, mutation=None):
    return lambda q, k, v, la, b, S0, erase, gate: oracle.chunkwise(q, k, v, la, b, S0, C=C, mutation=mutation,
                                                                   erase=erase, gate=gate)


VRUNNERS = {"recurrent": vrec(), "chunkwise_c1": vchk(1), "chunkwise_c5": vchk(5), "chunkwise_c16": vchk(16)}


@pytest.mark.parametrize("runner", list(VRUNNERS))
@pytest.mark.parametrize("pin", pins.VARIANT_PINS, ids=lambda p: p.__name__)
def test_variant_pins(pin, runner):
    assert pin(VRUNNERS[runner]) < TOL


@pytest.mark.parametrize("erase,gate", [(True, "scalar"), (True, "none"), (False, "channel"), (False, "scalar"),
                                        (False, "none")])
@pytest.mark.parametrize("C,T", [(1, 9), (4, 33), (16, 16), (64, 100)])
def test_variant_recurrence_equals_chunkwise(erase, gate, C, T):
    q, k, v, la, beta, S0 = pins.random_inputs(300 + T + C, T=T, dk=6, dv=5)
    g = {"channel": la, "scalar": la[..., 0], "none": None}[gate]
    o1, s1 = oracle.recurrent(q, k, v, g, beta, S0, erase=erase, gate=gate)
    o2, s2 = oracle.chunkwise(q, k, v, g, beta, S0, C=C, erase=erase, gate=gate)
    assert np.abs(o1 - o2).max() / max(1.0, np.abs(o1).max()) < 1e-12
    assert np.abs(s1 - s2).max() / max(1.0, np.abs(s1).max()) < 1e-12


@pytest.mark.parametrize("erase,gate", [(True, "scalar"), (False, "channel"), (False, "none")])
def test_variant_decode_chaining(erase, gate):
    """T single-token steps of the variant equal its prefill recurrence."""
    q, k, v, la, beta, S0 = pins.random_inputs(400, T=12, dk=6, dv=5)
    g = {"channel": la, "scalar": la[..., 0], "none": None}[gate]
    o_ref, S_ref = oracle.recurrent(q, k, v, g, beta, S0, erase=erase, gate=gate)
    S = S0
    for t in range(q.shape[1]):
        gt = None if g is None else g[:, t]
        o, S = oracle.decode_step(q[:, t], k[:, t], v[:, t], gt, beta[:, t], S, erase=erase, gate=gate)
        assert np.abs(o - o_ref[:, t]).max() < 1e-12
    assert np.abs(S - S_ref).max() < 1e-12


@pytest.mark.parametrize("mutation,pin", [("erase_always", pins.p12_gated_linear_attention),
                                          ("erase_always", pins.p13_plain_linear_attention),
                                          ("scalar_gate_twice", pins.p11_scalar_gated_delta)])
@pytest.mark.parametrize("runner", ["recurrent", "chunkwise"])
def test_variant_mutations_caught(mutation, pin, runner):
    run = vrec(mutation) if runner == "recurrent" else vchk(8, mutation)
    assert pin(run) > 1e-6


def test_variant_bad_switches():
    q, k, v, la, beta, S0 = pins.random_inputs(1, T=4, dk=4, dv=4)
    with pytest.raises(ValueError):
        oracle.recurrent(q, k, v, None, beta, S0, gate="channel")  # a gate needs log_alpha
    with pytest.raises(ValueError):
        oracle.chunkwise(q, k, v, la, beta, S0, C=4, gate=3)


def test_varlen_equal_lengths_equals_dense_batch():
    """Packing B equal-length sequences back to back is the dense [B, T] batch."""
    q, k, v, la, beta, S0 = pins.random_inputs(500, T=21, dk=6, dv=5, B_=3, H_=2)
    o_d, s_d = oracle.recurrent(q, k, v, la, beta, S0)
    pack = lambda x: x.reshape((-1,) + x.shape[2:])
    o_v, s_v = oracle.recurrent_varlen(pack(q), pack(k), pack(v), pack(la), pack(beta), [0, 21, 42, 63], S0)
    assert np.abs(o_v - pack(o_d)).max() < 1e-12 and np.abs(s_v - s_d).max() < 1e-12


def test_varlen_empty_sequence_keeps_state():
    q, k, v, la, beta, S0 = pins.random_inputs(501, T=10, dk=4, dv=4, B_=2, H_=1)
    pack = lambda x: x.reshape((-1,) + x.shape[2:])
    o_v, s_v = oracle.recurrent_varlen(pack(q), pack(k), pack(v), pack(la), pack(beta), [0, 0, 20], S0)
    assert np.array_equal(s_v[0], S0[0])
    o_1, s_1 = oracle.recurrent(q.reshape(1, 20, 1, 4), k.reshape(1, 20, 1, 4), v.reshape(1, 20, 1, 4),
                                la.reshape(1, 20, 1, 4), beta.reshape(1, 20, 1), S0[1:2])
    assert np.abs(s_v[1] - s_1[0]).max() < 1e-12


# ---------------------------------------------------------------- affine maps of token runs (chunk-parallel scan)


def _one_head(seed, T, dk=6, dv=5, la_range=(0.01, 1.0)):
    q, k, v, la, beta, S0 = pins.random_inputs(seed, T=T, dk=dk, dv=dv, la_range=la_range, B_=1, H_=1)
    return q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], beta[0, :, 0], S0[0, 0]


@pytest.mark.parametrize("erase,gate", [(True, "channel"), (True, "scalar"), (True, "none"), (False, "channel"),
                                        (False, "none")])
def test_affine_map_reproduces_recurrence(erase, gate):
    """M S0 + c equals the C recurrence's final state for several S0 (the map
    is the run's action on any state), and o is unaffected by the split."""
    q, k, v, la, beta, _ = _one_head(510, T=19)
    lag = {"channel": la, "scalar": la[:, 0], "none": None}[gate]
    M, c = oracle.segment_affine_map(k, v, lag, beta, erase=erase, gate=gate)
    r = np.random.default_rng(511)
    for _ in range(3):
        S0 = r.standard_normal((6, 5))
        x = lambda a: None if a is None else a[None, :, None]
        _, ST = oracle.recurrent(x(q), x(k), x(v), x(lag), x(beta), S0[None, None], erase=erase, gate=gate)
        assert np.abs(M @ S0 + c - ST[0, 0]).max() < 1e-12


def test_affine_map_closed_forms():
    """No erase: M = Diag(exp(sum log_alpha)) (identity without a gate) and
    c = sum_t exp(G_T - G_t) b_t k_t v_t^T. beta = 0 with erase: M is the pure
    decay and c = 0."""
    _, k, v, la, beta, _ = _one_head(512, T=11)
    M, c = oracle.segment_affine_map(k, v, la, beta, erase=False, gate="channel")
    G = np.cumsum(la, axis=0)
    assert np.abs(M - np.diag(np.exp(G[-1]))).max() < 1e-13
    c_ref = sum(beta[t] * np.outer(np.exp(G[-1] - G[t]) * k[t], v[t]) for t in range(11))
    assert np.abs(c - c_ref).max() < 1e-13
    M, c = oracle.segment_affine_map(k, v, None, beta, erase=False, gate="none")
    assert np.abs(M - np.eye(6)).max() == 0.0
    M, c = oracle.segment_affine_map(k, v, la, np.zeros_like(beta), erase=True, gate="channel")
    assert np.abs(M - np.diag(np.exp(G[-1]))).max() < 1e-13 and np.abs(c).max() == 0.0


def test_segment_scan_composes_to_whole_run():
    """Splitting a run into segments, scanning their maps from S0 and reading the
    last state equals the whole run's map applied to S0; every entry state is
    the recurrence's state at that segment boundary."""
    q, k, v, la, beta, S0 = _one_head(513, T=40)
    cuts = [0, 7, 8, 23, 40]
    maps = [oracle.segment_affine_map(k[a:b], v[a:b], la[a:b], beta[a:b]) for a, b in zip(cuts, cuts[1:])]
    states = oracle.segment_scan(maps, S0)
    M, c = oracle.segment_affine_map(k, v, la, beta)
    assert np.abs(states[-1] - (M @ S0 + c)).max() < 1e-12
    for j, t in enumerate(cuts[1:-1], start=1):
        _, St = oracle.recurrent(q[None, :t, None], k[None, :t, None], v[None, :t, None], la[None, :t, None],
                                 beta[None, :t, None], S0[None, None])
        assert np.abs(states[j] - St[0, 0]).max() < 1e-12


# ---------------------------------------------------------------- backward (gradients of the recurrence)


def _loss_and_grads(seed, erase, gate, T=5, dk=3, dv=2):
    q, k, v, la, beta, S0 = pins.random_inputs(seed, T=T, dk=dk, dv=dv, B_=1, H_=2)
    lag = {"channel": la, "scalar": la[..., 0], "none": None}[gate]
    r = np.random.default_rng(seed + 1)
    Wo = r.standard_normal(v.shape)
    WS = r.standard_normal(S0.shape)
    inputs = {"q": q, "k": k, "v": v, "log_alpha": lag, "beta": beta, "S0": S0}

    def loss(x):
        o, ST = oracle.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], erase=erase, gate=gate)
        return float((o * Wo).sum() + (ST * WS).sum())

    g = oracle.recurrent_bwd(q, k, v, lag, beta, S0, Wo, WS, erase=erase, gate=gate, ckpt=2)
    return inputs, loss, g


@pytest.mark.parametrize("erase,gate", [(True, "channel"), (True, "scalar"), (True, "none"), (False, "channel"),
                                        (False, "scalar"), (False, "none")])
def test_bwd_matches_finite_differences(erase, gate):
    """Every gradient element against a central difference of the forward
    oracle (a linear functional of o and S_T), for every variant."""
    inputs, loss, g = _loss_and_grads(520, erase, gate)
    names = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dlog_alpha", "beta": "dbeta", "S0": "dS0"}
    eps = 1e-6
    for name, gname in names.items():
        x = inputs[name]
        if x is None:
            assert g[gname] is None
            continue
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = {kk: (None if vv is None else vv.copy()) for kk, vv in inputs.items()}
            xm = {kk: (None if vv is None else vv.copy()) for kk, vv in inputs.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            fd[idx] = (loss(xp) - loss(xm)) / (2 * eps)
        assert np.abs(g[gname] - fd).max() < 1e-7 * max(1.0, np.abs(fd).max()), (name, erase, gate)


def test_bwd_linear_attention_closed_form():
    """No erase, no gate: o_t = S0^T q_t + sum_{s<=t} (q_t . k_s) b_s v_s and
    S_T = S0 + sum_s b_s k_s v_s^T, so dv_s = b_s (sum_{t>=s} (q_t . k_s) do_t
    + dS_T^T k_s) and dq_t = S0 do_t + sum_{s<=t} k_s b_s (v_s . do_t)."""
    q, k, v, _, beta, S0 = pins.random_inputs(521, T=9, dk=5, dv=4, B_=1, H_=1)
    r = np.random.default_rng(522)
    do = r.standard_normal(v.shape)
    dST = r.standard_normal(S0.shape)
    g = oracle.recurrent_bwd(q, k, v, None, beta, S0, do, dST, erase=False, gate="none", ckpt=4)
    Q, K, V, Bt, DO = q[0, :, 0], k[0, :, 0], v[0, :, 0], beta[0, :, 0], do[0, :, 0]
    for s in range(9):
        dv_ref = Bt[s] * (sum((Q[t] @ K[s]) * DO[t] for t in range(s, 9)) + dST[0, 0].T @ K[s])
        assert np.abs(g["dv"][0, s, 0] - dv_ref).max() < 1e-12
        dq_ref = S0[0, 0] @ DO[s] + sum(K[u] * Bt[u] * (V[u] @ DO[s]) for u in range(s + 1))
        assert np.abs(g["dq"][0, s, 0] - dq_ref).max() < 1e-12
    assert np.abs(g["dS0"][0, 0] - (dST[0, 0] + Q.T @ DO)).max() < 1e-12


def test_bwd_checkpoint_interval_invariant():
    q, k, v, la, beta, S0 = pins.random_inputs(523, T=13, dk=4, dv=3, B_=1, H_=2)
    do = np.random.default_rng(524).standard_normal(v.shape)
    a = oracle.recurrent_bwd(q, k, v, la, beta, S0, do, ckpt=1)
    b = oracle.recurrent_bwd(q, k, v, la, beta, S0, do, ckpt=64)
    for n in a:
        assert np.array_equal(a[n], b[n])


# ---------------------------------------------------------------- planted mistakes in the Python oracle functions


@pytest.mark.parametrize("mutation", oracle.BWD_MUTATIONS)
def test_bwd_pins_catch_planted_mistakes(mutation):
    """Each planted mistake in the backward oracle breaks the finite-difference
    pin (in at least one variant)."""
    caught = False
    for erase, gate in [(True, "channel"), (True, "scalar")]:
        q, k, v, la, beta, S0 = pins.random_inputs(530, T=5, dk=3, dv=2, B_=1, H_=1)
        lag = la if gate == "channel" else la[..., 0]
        r = np.random.default_rng(531)
        Wo, WS = r.standard_normal(v.shape), r.standard_normal(S0.shape)
        g = oracle.recurrent_bwd(q, k, v, lag, beta, S0, Wo, WS, erase=erase, gate=gate, mutation=mutation)
        inputs = {"q": q, "k": k, "v": v, "log_alpha": lag, "beta": beta, "S0": S0}
        names = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dlog_alpha", "beta": "dbeta", "S0": "dS0"}
        for name, gname in names.items():
            x = inputs[name]
            fd = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp = {kk: vv.copy() for kk, vv in inputs.items()}
                xm = {kk: vv.copy() for kk, vv in inputs.items()}
                xp[name][idx] += 1e-6
                xm[name][idx] -= 1e-6
                lp = oracle.recurrent(xp["q"], xp["k"], xp["v"], xp["log_alpha"], xp["beta"], xp["S0"], gate=gate)
                lm = oracle.recurrent(xm["q"], xm["k"], xm["v"], xm["log_alpha"], xm["beta"], xm["S0"], gate=gate)
                fd[idx] = ((lp[0] * Wo).sum() + (lp[1] * WS).sum() - (lm[0] * Wo).sum() - (lm[1] * WS).sum()) / 2e-6
            if np.abs(g[gname] - fd).max() > 1e-5:
                caught = True
    assert caught, mutation


@pytest.mark.parametrize("mutation", oracle.AFFINE_MUTATIONS)
def test_affine_pins_catch_planted_mistakes(mutation):
    q, k, v, la, beta, _ = _one_head(532, T=9)
    M, c = oracle.segment_affine_map(k, v, la, beta, mutation=mutation)
    S0 = np.random.default_rng(533).standard_normal((6, 5))
    _, ST = oracle.recurrent(q[None, :, None], k[None, :, None], v[None, :, None], la[None, :, None],
                             beta[None, :, None], S0[None, None])
    assert np.abs(M @ S0 + c - ST[0, 0]).max() > 1e-6, mutation


@pytest.mark.parametrize("mutation", oracle.VARLEN_MUTATIONS)
def test_varlen_pins_catch_planted_mistakes(mutation):
    q, k, v, la, beta, S0 = pins.random_inputs(534, T=21, dk=6, dv=5, B_=3, H_=2)
    o_d, s_d = oracle.recurrent(q, k, v, la, beta, S0)
    pack = lambda x: x.reshape((-1,) + x.shape[2:])
    o_v, s_v = oracle.recurrent_varlen(pack(q), pack(k), pack(v), pack(la), pack(beta), [0, 21, 42, 63], S0,
                                       mutation=mutation)
    assert max(np.abs(o_v - pack(o_d)).max(), np.abs(s_v - s_d).max()) > 1e-6, mutation
