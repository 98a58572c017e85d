"""KDA oracle (test infrastructure only).

A plain fp64 CPU implementation of the fine-grained gated delta rule, written
in C (``kda_oracle.c``) and called here through ctypes. Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs
use it; the product package never imports it, and it never imports the
product package.

Sources followed: "Decoding Hybrid Attention Architectures" section 3.4 (the
KDA update and the variant table: the erase / gate switches select the delta
rule, the scalar gated delta rule and the additive-write family), section 3.2
(role of beta), section 4 (the chunkwise form); "Technical Analysis ... Novel Hybrid Linear Attention"
sections 2.4 and 3.1-3.2. Every function is pinned by tests/test_oracle.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Planted-mistake selectors (mirror the enum in kda_oracle.c); 0 = correct.
MUTATIONS = {
    "no_decay": 1,
    "decay_after": 2,
    "erase_sign": 3,
    "read_before": 4,
    "transposed_read": 5,
    "beta_write_only": 6,
    "decay_columns": 7,
    "prefix_decay_k": 8,
    "strict_tril_o": 9,
    "erase_always": 10,
    "scalar_gate_twice": 11,
}

# Variant switches (see kda_oracle.c): erase 1 = delta-rule family, 0 = additive
# write; gate 0 = per-channel log_alpha [.., dk], 1 = one per token and head, 2 = none.
GATES = {"channel": 0, "scalar": 1, "none": 2}


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (plain C11, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC,
                               "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.kda_oracle_recurrent.argtypes = [P] * 8 + [I] * 7
        lib.kda_oracle_recurrent.restype = I
        lib.kda_oracle_chunkwise.argtypes = [P] * 8 + [I] * 6 + [P, P, I, I]
        lib.kda_oracle_chunkwise.restype = I
        lib.kda_oracle_decode_step.argtypes = [P] * 8 + [I] * 5
        lib.kda_oracle_decode_step.restype = I
        lib.kda_oracle_recurrent_v.argtypes = [P] * 8 + [I] * 9
        lib.kda_oracle_recurrent_v.restype = I
        lib.kda_oracle_chunkwise_v.argtypes = [P] * 8 + [I] * 6 + [P, P, I, I, I, I]
        lib.kda_oracle_chunkwise_v.restype = I
        lib.kda_oracle_decode_step_v.argtypes = [P] * 8 + [I] * 7
        lib.kda_oracle_decode_step_v.restype = I
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor -> numpy, no arithmetic
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _gate(gate):
    return GATES[gate] if isinstance(gate, str) else int(gate)


def recurrent(q, k, v, log_alpha, beta, S0=None, nthreads: int = 0, mutation: str | None = None,
              erase: bool = True, gate="channel"):
    """Token-by-token fp64 recurrence. Shapes: q,k [B,T,H,dk]; log_alpha
    [B,T,H,dk] (gate "channel"), [B,T,H] (gate "scalar") or None (gate
    "none"); v [B,T,H,dv]; beta [B,T,H]; S0 [B,H,dk,dv] or None. erase=False
    selects the additive-write family. Returns (o, S_T)."""
    q, k, v, la, beta, S0 = map(_f64, (q, k, v, log_alpha, beta, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    rc = _load().kda_oracle_recurrent_v(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta), _ptr(S0),
                                        _ptr(o), _ptr(ST), B, T, H, dk, dv, int(bool(erase)), _gate(gate),
                                        nthreads, MUTATIONS[mutation] if mutation else 0)
    if rc:
        raise ValueError("kda_oracle_recurrent_v: bad sizes or switches")
    return o, ST


def chunkwise(q, k, v, log_alpha, beta, S0=None, C: int = 64, nthreads: int = 0,
              mutation: str | None = None, debug: bool = False, erase: bool = True, gate="channel"):
    """fp64 chunkwise reformulation. Returns (o, S_T) or, with debug=True,
    (o, S_T, A, Tinv) where A and Tinv are [B,H,NC,C,C]."""
    q, k, v, la, beta, S0 = map(_f64, (q, k, v, log_alpha, beta, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    NC = (T + C - 1) // C
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    A = np.zeros((B, H, NC, C, C)) if debug else None
    Ti = np.zeros((B, H, NC, C, C)) if debug else None
    rc = _load().kda_oracle_chunkwise_v(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta), _ptr(S0),
                                        _ptr(o), _ptr(ST), B, T, H, dk, dv, C, _ptr(A), _ptr(Ti),
                                        int(bool(erase)), _gate(gate), nthreads,
                                        MUTATIONS[mutation] if mutation else 0)
    if rc:
        raise ValueError("kda_oracle_chunkwise_v: bad sizes or switches")
    return (o, ST, A, Ti) if debug else (o, ST)


def decode_step(q, k, v, log_alpha, beta, S, nthreads: int = 0, erase: bool = True, gate="channel"):
    """One recurrent step for [N,H,*] inputs and state S [N,H,dk,dv]
    (log_alpha [N,H,dk], [N,H] or None by gate). Returns (o, S_new)."""
    q, k, v, la, beta, S = map(_f64, (q, k, v, log_alpha, beta, S))
    N, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((N, H, dv))
    Sn = np.zeros((N, H, dk, dv))
    rc = _load().kda_oracle_decode_step_v(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta), _ptr(S),
                                          _ptr(Sn), _ptr(o), N, H, dk, dv, int(bool(erase)), _gate(gate),
                                          nthreads)
    if rc:
        raise ValueError("kda_oracle_decode_step_v: bad sizes or switches")
    return o, Sn


def recurrent_varlen(q, k, v, log_alpha, beta, cu_seqlens, S0=None, erase: bool = True, gate="channel",
                     mutation: str | None = None):
    """Packed variable-length sequences: q,k [total_T,H,dk], v [total_T,H,dv],
    beta [total_T,H], log_alpha [total_T,H,dk] / [total_T,H] / None, cu_seqlens
    [N+1] offsets, S0 [N,H,dk,dv] or None. Each sequence is its own recurrence
    (the definition of packing); returns (o [total_T,H,dv], S_T [N,H,dk,dv])."""
    q, k, v, la, beta, S0 = map(_f64, (q, k, v, log_alpha, beta, S0))
    cu = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    N = len(cu) - 1
    H, dk = q.shape[1], q.shape[2]
    dv = v.shape[-1]
    o = np.zeros((q.shape[0], H, dv))
    ST = np.zeros((N, H, dk, dv))
    for n in range(N):
        a, b = cu[n], cu[n + 1]
        s0 = None if S0 is None else S0[n:n + 1]
        if mutation == "state_leaks_between_sequences" and n > 0:
            s0 = ST[n - 1:n]
        if b == a:
            ST[n] = 0.0 if S0 is None else S0[n]
            continue
        sl = (lambda x: None if x is None else x[None, a:b])
        on, sn = recurrent(sl(q), sl(k), sl(v), sl(la), sl(beta), s0, erase=erase, gate=gate)
        o[a:b] = on[0]
        ST[n] = sn[0]
    return o, ST


def segment_affine_map(k, v, log_alpha, beta, erase: bool = True, gate="channel", mutation: str | None = None):
    """The update is affine in the state ("Decoding Hybrid Attention
    Architectures" section 3.4: S_t = A_t S_{t-1} + b_t k_t v_t^T with
    A_t = (I - e b_t k_t k_t^T) Diag(a_t)), so a run of tokens maps S_in to
    M S_in + c. One head, fp64, explicit matrices: k [T,dk], v [T,dv], beta [T],
    log_alpha [T,dk] / [T] / None by gate. Returns (M [dk,dk], c [dk,dv])."""
    k, v, beta = _f64(k), _f64(v), _f64(beta)
    la = _f64(log_alpha)
    T, dk = k.shape
    dv = v.shape[1]
    M = np.eye(dk)
    c = np.zeros((dk, dv))
    for t in range(T):
        if gate == "channel":
            a = np.exp(la[t])
        elif gate == "scalar":
            a = np.full(dk, np.exp(la[t]))
        else:
            a = np.ones(dk)
        A = np.diag(a)
        if erase:
            A = (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ A
        M = M @ A if mutation == "map_order_swapped" else A @ M
        if mutation == "write_before_erase":
            c = A @ (c + beta[t] * np.outer(k[t], v[t]))
        else:
            c = A @ c + beta[t] * np.outer(k[t], v[t])
    return M, c


def segment_scan(maps, S0):
    """States entering each segment from the segments' affine maps:
    S_in[0] = S0, S_in[j+1] = M_j S_in[j] + c_j. Returns the list of P+1
    states (the last is the final state)."""
    S = [np.asarray(S0, dtype=np.float64)]
    for M, c in maps:
        S.append(M @ S[-1] + c)
    return S


# Planted mistakes in the Python oracle functions, used only by the mutation
# tests (each must make a pin fail); None = correct.
BWD_MUTATIONS = ("no_read_key_grad", "decay_before_erase", "lam_for_lam_tilde", "beta_missing_in_dv")
AFFINE_MUTATIONS = ("write_before_erase", "map_order_swapped")
VARLEN_MUTATIONS = ("state_leaks_between_sequences",)


def recurrent_bwd(q, k, v, log_alpha, beta, S0, do, dST=None, erase: bool = True, gate="channel",
                  ckpt: int = 64, mutation: str | None = None):
    """Gradients of the token recurrence, by reverse-mode differentiation of
    each step (the pages give no backward pass; this is the chain rule applied
    to the update of "Decoding Hybrid Attention Architectures" section 3.4).

    Loss L with dL/do = do [B,T,H,dv] and dL/dS_T = dST [B,H,dk,dv] (None:
    0). Per step, with Lam = dL/dS_t (the future part plus q_t do_t^T):
        S~ = Diag(a_t) S_{t-1},  r = v_t - S~^T k_t,  delta = b_t r  (no erase: b_t v_t)
        dq_t = S_t do_t,  g = Lam^T k_t,  dv_t = b_t g,  db_t = g . r (no erase: g . v_t)
        dk_t = Lam delta - b_t S~ g   (second term only with the erase term)
        Lam~ = Lam - b_t k_t g^T      (dL/dS~; no erase: Lam)
        dlog_a_t = rowsum(Lam~ * S~)  (per channel; summed for a scalar gate)
        dL/dS_{t-1} = Diag(a_t) Lam~
    and dS0 = dL/dS_0. States are recomputed from checkpoints every `ckpt`
    tokens (same arithmetic, less memory). fp64 numpy; small cases only.
    Returns dict dq, dk, dv, dlog_alpha (shape of log_alpha, None without a
    gate), dbeta, dS0."""
    q, k, v, beta, do = map(_f64, (q, k, v, beta, do))
    la = _f64(log_alpha)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S0 = np.zeros((B, H, dk, dv)) if S0 is None else _f64(S0)
    dST = np.zeros((B, H, dk, dv)) if dST is None else _f64(dST)
    out = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dbeta", beta))}
    out["dlog_alpha"] = None if gate == "none" else np.zeros_like(la)
    out["dS0"] = np.zeros_like(S0)

    def decay(b, t, h):
        if gate == "channel":
            return np.exp(la[b, t, h])
        if gate == "scalar":
            return np.full(dk, np.exp(la[b, t, h]))
        return np.ones(dk)

    def step(S, b, t, h):
        St = decay(b, t, h)[:, None] * S
        r = v[b, t, h] - St.T @ k[b, t, h]
        delta = beta[b, t, h] * (r if erase else v[b, t, h])
        return St, r, St + np.outer(k[b, t, h], delta)

    for b in range(B):
        for h in range(H):
            # forward: states at the checkpoints
            marks = {}
            S = S0[b, h].copy()
            for t in range(T):
                if t % ckpt == 0:
                    marks[t] = S.copy()
                S = step(S, b, t, h)[2]
            Lam = dST[b, h].copy()
            for t0 in sorted(marks, reverse=True):
                t1 = min(t0 + ckpt, T)
                prev = [marks[t0]]
                for t in range(t0, t1 - 1):
                    prev.append(step(prev[-1], b, t, h)[2])
                for t in range(t1 - 1, t0 - 1, -1):
                    St, r, S_t = step(prev[t - t0], b, t, h)
                    kt, bt = k[b, t, h], beta[b, t, h]
                    Lam = Lam + np.outer(q[b, t, h], do[b, t, h])
                    out["dq"][b, t, h] = S_t @ do[b, t, h]
                    g = Lam.T @ kt
                    delta = bt * (r if erase else v[b, t, h])
                    out["dv"][b, t, h] = (1.0 if mutation == "beta_missing_in_dv" else bt) * g
                    out["dbeta"][b, t, h] = g @ (r if erase else v[b, t, h])
                    read = bt * (St @ g) if erase and mutation != "no_read_key_grad" else 0.0
                    out["dk"][b, t, h] = Lam @ delta - read
                    Lt = Lam - bt * np.outer(kt, g) if erase else Lam
                    Ld = Lam if mutation == "lam_for_lam_tilde" else Lt
                    if gate == "channel":
                        out["dlog_alpha"][b, t, h] = (Ld * St).sum(axis=1)
                    elif gate == "scalar":
                        out["dlog_alpha"][b, t, h] = (Ld * St).sum()
                    if mutation == "decay_before_erase" and erase:
                        La = decay(b, t, h)[:, None] * Lam
                        Lam = La - bt * np.outer(kt, La.T @ kt)
                    else:
                        Lam = decay(b, t, h)[:, None] * Lt
            out["dS0"][b, h] = Lam
    return out
