"""Pins for the KDA oracle: checks fixed by the pages and by mathematics, not
by the oracle itself. Each pin takes a `run(q, k, v, log_alpha, beta, S0) ->
(o, S_T)` callable on fp64 numpy arrays ([B,T,H,d] layouts) and returns the
max abs deviation from the value the pin fixes.

Sources: "Decoding Hybrid Attention Architectures" sections 3.1 (pure linear
attention), 3.2 (delta rule; beta = 1 with normalised keys overwrites the
slot), 3.3 (scalar-gated delta), 3.4 (fine-grained gate, variant table).
"""
from __future__ import annotations

import numpy as np

B, H = 1, 2


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def random_inputs(seed, T=24, dk=8, dv=8, la_range=(0.01, 1.0), s0=True, B_=B, H_=H):
    r = _rng(seed)
    q = _unit(r.standard_normal((B_, T, H_, dk)))
    k = _unit(r.standard_normal((B_, T, H_, dk)))
    v = r.standard_normal((B_, T, H_, dv))
    la = -r.uniform(*la_range, (B_, T, H_, dk))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((B_, T, H_))))
    S0 = r.standard_normal((B_, H_, dk, dv)) if s0 else None
    return q, k, v, la, beta, S0


def p1_identity(run, seed=11, T=24, dk=8, dv=8):
    """alpha = 1, beta = 0: nothing is erased or written, so S_t = S_0 and
    o_t = S_0^T q_t exactly."""
    q, k, v, la, beta, S0 = random_inputs(seed, T, dk, dv)
    la[:] = 0.0
    beta[:] = 0.0
    o, ST = run(q, k, v, la, beta, S0)
    o_ref = np.einsum("bhij,bthi->bthj", S0, q)
    return max(np.abs(ST - S0).max(), np.abs(o - o_ref).max())


def p2_linear_attention(run, seed=12, T=8, dk=8, dv=8):
    """Section 3.1: with alpha = 1, beta = 1, S_0 = 0 and mutually orthogonal
    unit keys (distinct basis vectors), the erase term vanishes, so the state is
    the plain linear-attention sum S_t = sum_{s<=t} k_s v_s^T and
    o_t = sum_{s<=t} (q_t . k_s) v_s."""
    assert T <= dk
    r = _rng(seed)
    q, k, v, la, beta, _ = random_inputs(seed, T, dk, dv)
    la[:] = 0.0
    beta[:] = 1.0
    k[:] = 0.0
    for b in range(k.shape[0]):
        for h in range(k.shape[2]):
            perm = r.permutation(dk)[:T]
            for t in range(T):
                k[b, t, h, perm[t]] = 1.0
    o, ST = run(q, k, v, la, beta, None)
    err = 0.0
    for b in range(k.shape[0]):
        for h in range(k.shape[2]):
            S = np.zeros((dk, dv))
            for t in range(T):
                S = S + np.outer(k[b, t, h], v[b, t, h])
                o_ref = sum((q[b, t, h] @ k[b, s, h]) * v[b, s, h] for s in range(t + 1))
                err = max(err, np.abs(o[b, t, h] - o_ref).max())
            err = max(err, np.abs(ST[b, h] - S).max())
    return err


def p3_pure_decay(run, seed=13, T=24, dk=8, dv=8):
    """beta = 0: only the gate acts, S_t = Diag(exp(sum_{s<=t} log_alpha_s)) S_0
    (row i scaled by the product of alpha_i over the steps so far)."""
    q, k, v, la, beta, S0 = random_inputs(seed, T, dk, dv)
    beta[:] = 0.0
    o, ST = run(q, k, v, la, beta, S0)
    cum = np.cumsum(la, axis=1)                    # [B,T,H,dk]
    St = np.exp(cum)[..., None] * S0[:, None]      # [B,T,H,dk,dv]
    o_ref = np.einsum("bthij,bthi->bthj", St, q)
    return max(np.abs(ST - St[:, -1]).max(), np.abs(o - o_ref).max())


def p4_retrieval(run, seed=14, T=24, dk=8, dv=8):
    """Section 3.2: with unit-norm k_t and beta_t = 1 the update overwrites the
    slot, so S_t^T k_t = v_t whatever S_{t-1} and the gate were. Reading with
    q_t = k_t must return v_t."""
    q, k, v, la, beta, S0 = random_inputs(seed, T, dk, dv)
    beta[:] = 1.0
    q = k.copy()
    o, _ = run(q, k, v, la, beta, S0)
    return np.abs(o - v).max()


def p5_scalar_gate(run, seed=15, T=24, dk=8, dv=8):
    """Section 3.3: when every channel shares one gate a_t, the fine-grained
    rule is the scalar-gated delta rule S_t = a_t (I - b_t k_t k_t^T) S_{t-1}
    + b_t k_t v_t^T. Compared with that rule written with explicit matrices."""
    q, k, v, la, beta, S0 = random_inputs(seed, T, dk, dv)
    la[:] = la[..., :1]
    o, ST = run(q, k, v, la, beta, S0)
    err = 0.0
    I = np.eye(dk)
    for b in range(q.shape[0]):
        for h in range(q.shape[2]):
            S = S0[b, h].copy()
            for t in range(T):
                a = np.exp(la[b, t, h, 0])
                kt, bt = k[b, t, h], beta[b, t, h]
                S = a * (I - bt * np.outer(kt, kt)) @ S + bt * np.outer(kt, v[b, t, h])
                err = max(err, np.abs(o[b, t, h] - S.T @ q[b, t, h]).max())
            err = max(err, np.abs(ST[b, h] - S).max())
    return err


ALL_PINS = [p1_identity, p2_linear_attention, p3_pure_decay, p4_retrieval, p5_scalar_gate]


# ---------------------------------------------------------------- variants
# Each variant pin takes `run(q, k, v, log_alpha, beta, S0, erase=..., gate=...)`
# and compares with the rule as the pages state it, written out independently.


def p10_delta_rule(run, seed=20, T=24, dk=8, dv=8):
    """Section 3.2 (delta rule, no gate): S_t = (I - b_t k_t k_t^T) S_{t-1}
    + b_t k_t v_t^T, with explicit matrices."""
    q, k, v, _, beta, S0 = random_inputs(seed, T, dk, dv)
    o, ST = run(q, k, v, None, beta, S0, erase=True, gate="none")
    err = 0.0
    I = np.eye(dk)
    for b in range(q.shape[0]):
        for h in range(q.shape[2]):
            S = S0[b, h].copy()
            for t in range(T):
                kt, bt = k[b, t, h], beta[b, t, h]
                S = (I - bt * np.outer(kt, kt)) @ S + bt * np.outer(kt, v[b, t, h])
                err = max(err, np.abs(o[b, t, h] - S.T @ q[b, t, h]).max())
            err = max(err, np.abs(ST[b, h] - S).max())
    return err


def p11_scalar_gated_delta(run, seed=21, T=24, dk=8, dv=8):
    """Section 3.3 / variant table (scalar gated delta, one gate per token and
    head): S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T, the scalar
    applied outside the erase as printed, with explicit matrices."""
    q, k, v, la, beta, S0 = random_inputs(seed, T, dk, dv)
    g = la[..., 0]                                  # [B,T,H]
    o, ST = run(q, k, v, g, beta, S0, erase=True, gate="scalar")
    err = 0.0
    I = np.eye(dk)
    for b in range(q.shape[0]):
        for h in range(q.shape[2]):
            S = S0[b, h].copy()
            for t in range(T):
                kt, bt = k[b, t, h], beta[b, t, h]
                S = np.exp(g[b, t, h]) * (I - bt * np.outer(kt, kt)) @ S + bt * np.outer(kt, v[b, t, h])
                err = max(err, np.abs(o[b, t, h] - S.T @ q[b, t, h]).max())
            err = max(err, np.abs(ST[b, h] - S).max())
    return err


def p12_gated_linear_attention(run, seed=22, T=24, dk=8, dv=8):
    """Per-dimension gated linear attention (named beside the variant table):
    S_t = Diag(a_t) S_{t-1} + b_t k_t v_t^T, so in closed form
    S_t = Diag(e^{G_t}) S_0 + sum_{s<=t} b_s Diag(e^{G_t - G_s}) k_s v_s^T with
    G_t = sum_{u<=t} log a_u, and o_t = S_t^T q_t."""
    q, k, v, la, beta, S0 = random_inputs(seed, T, dk, dv)
    o, ST = run(q, k, v, la, beta, S0, erase=False, gate="channel")
    G = np.cumsum(la, axis=1)                       # [B,T,H,dk]
    err = 0.0
    for b in range(q.shape[0]):
        for h in range(q.shape[2]):
            for t in range(T):
                S = np.exp(G[b, t, h])[:, None] * S0[b, h]
                for s_ in range(t + 1):
                    S = S + beta[b, s_, h] * np.outer(np.exp(G[b, t, h] - G[b, s_, h]) * k[b, s_, h], v[b, s_, h])
                err = max(err, np.abs(o[b, t, h] - S.T @ q[b, t, h]).max())
                if t == T - 1:
                    err = max(err, np.abs(ST[b, h] - S).max())
    return err


def p13_plain_linear_attention(run, seed=23, T=24, dk=8, dv=8):
    """Section 3.1: S_t = S_{t-1} + k_t v_t^T (no erase, no gate, b = 1):
    o_t = S_0^T q_t + sum_{s<=t} (q_t . k_s) v_s and S_T = S_0 + sum_s k_s v_s^T,
    for any keys (not only orthogonal ones)."""
    q, k, v, _, beta, S0 = random_inputs(seed, T, dk, dv)
    beta[:] = 1.0
    o, ST = run(q, k, v, None, beta, S0, erase=False, gate="none")
    err = 0.0
    for b in range(q.shape[0]):
        for h in range(q.shape[2]):
            for t in range(T):
                o_ref = S0[b, h].T @ q[b, t, h] + sum((q[b, t, h] @ k[b, s_, h]) * v[b, s_, h] for s_ in range(t + 1))
                err = max(err, np.abs(o[b, t, h] - o_ref).max())
            err = max(err, np.abs(ST[b, h] - (S0[b, h] + k[b, :, h].T @ v[b, :, h])).max())
    return err


VARIANT_PINS = [p10_delta_rule, p11_scalar_gated_delta, p12_gated_linear_attention, p13_plain_linear_attention]
