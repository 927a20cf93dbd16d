"""Pins for the fp64 oracle: results the mathematics fixes independently of it.

Each pin runs the oracle (``lib``: a loaded oracle library, by default the real
one) on a small seeded case and returns the largest relative error against a
value computed another way.  The tests assert each error is at rounding level;
the mutation test runs the same pins against deliberately broken copies of the
oracle and asserts that every planted mistake makes at least one pin fail.
"""
from __future__ import annotations

import itertools
import json
import os

import numpy as np

import oracle
from oracle.deferred import DeferredHead

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rel(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = max(np.linalg.norm(ref), 1e-300)
    return float(np.linalg.norm(x - ref) / den)


def _case(seed, T, dk, dv, decay, update, n=3, lam_scale=0.3, unit_k=False):
    r = np.random.default_rng(seed)
    S0 = r.standard_normal((n, dk, dv))
    q = r.standard_normal((n, T, dk))
    k = r.standard_normal((n, T, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((n, T, dv))
    lam = None
    if decay == "scalar":
        lam = -lam_scale * r.random((n, T))
    elif decay == "diag":
        lam = -lam_scale * r.random((n, T, dk))
    beta = r.random((n, T)) if update != "add" else None
    return S0, q, k, v, lam, beta


# --------------------------------------------------------------------------
# 1. additive, no decay: causal linear attention in its parallel form
#    O = Q S0 + tril(Q K^T) V  and  S_T = S0 + K^T V
#    (paper, "Background": the state aggregates the prefix's key-value products)
# --------------------------------------------------------------------------
def pin_additive_prefix_sum(lib=None):
    T, dk, dv = 9, 3, 5
    S0, q, k, v, _, _ = _case(11, T, dk, dv, "none", "add")
    out, S = oracle.eager_tasks(S0, q, k, v, None, None, decay="none", update="add",
                                ckpts=[T], lib=lib)
    err = 0.0
    for i in range(S0.shape[0]):
        Q, K, V = q[i], k[i], v[i]
        O_ref = Q @ S0[i] + np.tril(Q @ K.T) @ V
        S_ref = S0[i] + K.T @ V
        err = max(err, _rel(out[i], O_ref), _rel(S[i, 0], S_ref))
    return err


# --------------------------------------------------------------------------
# 2. additive, per-key decay: the unrolled recurrence
#    S_t[r,:] = e^{P_t[r]} S0[r,:] + sum_{i<=t} e^{P_t[r]-P_i[r]} k_i[r] v_i,
#    P_t = sum_{j<=t} lambda_j  (gated linear attention's parallel form)
# --------------------------------------------------------------------------
def pin_diag_decay_unrolled(lib=None):
    T, dk, dv = 8, 4, 3
    S0, q, k, v, lam, _ = _case(12, T, dk, dv, "diag", "add")
    out, S = oracle.eager_tasks(S0, q, k, v, lam, None, decay="diag", update="add",
                                ckpts=[T], lib=lib)
    err = 0.0
    for i in range(S0.shape[0]):
        P = np.cumsum(lam[i], axis=0)                     # [T, dk]
        O_ref = np.zeros((T, dv))
        for t in range(T):
            qt = q[i, t]
            O_ref[t] = (qt * np.exp(P[t])) @ S0[i]
            for j in range(t + 1):
                w = np.dot(qt * np.exp(P[t] - P[j]), k[i, j])
                O_ref[t] += w * v[i, j]
        S_ref = np.exp(P[-1])[:, None] * S0[i]
        for j in range(T):
            S_ref += np.outer(np.exp(P[-1] - P[j]) * k[i, j], v[i, j])
        err = max(err, _rel(out[i], O_ref), _rel(S[i, 0], S_ref))
    return err


# --------------------------------------------------------------------------
# 3. additive, constant scalar decay gamma: RetNet's parallel retention
#    O = (Q K^T * D) V + gamma^t Q S0,  D[t,i] = gamma^(t-i) for i <= t, else 0
# --------------------------------------------------------------------------
def pin_retention_parallel(lib=None):
    T, dk, dv = 10, 4, 4
    S0, q, k, v, _, _ = _case(13, T, dk, dv, "none", "add", n=2)
    gam = np.array([0.9, 0.75])
    lam = np.log(gam)[:, None] * np.ones((2, T))
    out, _ = oracle.eager_tasks(S0, q, k, v, lam, None, decay="scalar", update="add", lib=lib)
    err = 0.0
    tt = np.arange(T)
    for i in range(2):
        D = np.where(tt[:, None] >= tt[None, :], gam[i] ** (tt[:, None] - tt[None, :]), 0.0)
        O_ref = ((q[i] @ k[i].T) * D) @ v[i] + (gam[i] ** (tt + 1))[:, None] * (q[i] @ S0[i])
        err = max(err, _rel(out[i], O_ref))
    return err


# --------------------------------------------------------------------------
# 4. delta rule with explicit matrices (tiny d):
#    decayed reading   S_t = (I - beta k k^T) Diag(g) S_{t-1} + beta k v^T
#    undecayed reading S_t = (Diag(g) - beta k k^T) S_{t-1} + beta k v^T
# --------------------------------------------------------------------------
def pin_delta_matrix_form(lib=None):
    err = 0.0
    for decay, upd in itertools.product(("none", "scalar", "diag"), ("delta", "delta_undecayed")):
        T, dk, dv = 7, 3, 4
        S0, q, k, v, lam, beta = _case(14, T, dk, dv, decay, upd)
        out, S = oracle.eager_tasks(S0, q, k, v, lam, beta, decay=decay, update=upd,
                                    ckpts=[T], lib=lib)
        for i in range(S0.shape[0]):
            Sm = S0[i].copy()
            O_ref = np.zeros((T, dv))
            for t in range(T):
                if decay == "none":
                    G = np.eye(dk)
                elif decay == "scalar":
                    G = np.exp(lam[i, t]) * np.eye(dk)
                else:
                    G = np.diag(np.exp(lam[i, t]))
                kk = np.outer(k[i, t], k[i, t])
                if upd == "delta":
                    Sm = (np.eye(dk) - beta[i, t] * kk) @ G @ Sm
                else:
                    Sm = (G - beta[i, t] * kk) @ Sm
                Sm = Sm + beta[i, t] * np.outer(k[i, t], v[i, t])
                O_ref[t] = Sm.T @ q[i, t]
            err = max(err, _rel(out[i], O_ref), _rel(S[i, 0], Sm))
    return err


# --------------------------------------------------------------------------
# 5. delta-rule invariants
#    beta = 1, |k| = 1  =>  S_t^T k_t = v_t (the state recalls the written value)
#    beta = 0           =>  pure decay S_t = Diag(g) S_{t-1}
# --------------------------------------------------------------------------
def pin_delta_invariants(lib=None):
    err = 0.0
    T, dk, dv = 6, 5, 3
    for decay in ("none", "scalar", "diag"):
        S0, q, k, v, lam, _ = _case(15, T, dk, dv, decay, "delta", unit_k=True)
        ones = np.ones((S0.shape[0], T))
        _, S = oracle.eager_tasks(S0, q, k, v, lam, ones, decay=decay, update="delta",
                                  ckpts=list(range(1, T + 1)), lib=lib)
        for i in range(S0.shape[0]):
            for t in range(T):
                err = max(err, _rel(S[i, t].T @ k[i, t], v[i, t]))
        zeros = np.zeros((S0.shape[0], T))
        _, S = oracle.eager_tasks(S0, q, k, v, lam, zeros, decay=decay, update="delta",
                                  ckpts=[T], lib=lib)
        for i in range(S0.shape[0]):
            if decay == "none":
                tot = np.zeros(dk)
            elif decay == "scalar":
                tot = np.full(dk, lam[i].sum())
            else:
                tot = lam[i].sum(axis=0)
            err = max(err, _rel(S[i, 0], np.exp(tot)[:, None] * S0[i]))
    return err


# --------------------------------------------------------------------------
# 6. base + log (deferred, independent implementation of the paper's logical state)
#    equals eager at every step for every merge interval
# --------------------------------------------------------------------------
def pin_deferred_equals_eager(lib=None, caps=(1, 2, 3, 4, 8, 16, 32)):
    err = 0.0
    T, dk, dv = 40, 4, 3
    for decay, upd in itertools.product(("none", "scalar", "diag"),
                                        ("add", "delta", "delta_undecayed")):
        S0, q, k, v, lam, beta = _case(16, T, dk, dv, decay, upd, n=1, lam_scale=0.2)
        out, S = oracle.eager_tasks(S0, q, k, v, lam, beta, decay=decay, update=upd,
                                    ckpts=[T], lib=lib)
        for L in caps:
            h = DeferredHead(S0[0], L, decay, upd)
            O = np.array([h.decode(q[0, t], k[0, t], v[0, t],
                                   None if lam is None else lam[0, t],
                                   None if beta is None else beta[0, t]) for t in range(T)])
            err = max(err, _rel(O, out[0]), _rel(h.logical(), S[0, 0]))
    return err


# --------------------------------------------------------------------------
# 7. hand-derived scalar recurrences (d_k = d_v = 1), tests/golden
# --------------------------------------------------------------------------
def pin_scalar_golden(lib=None):
    with open(os.path.join(GOLDEN, "scalar_recurrence.json")) as f:
        cases = json.load(f)["cases"]
    err = 0.0
    for c in cases:
        T = len(c["q"])
        a = lambda key: np.asarray(c[key], np.float64).reshape(1, T, 1)
        lam = None
        if c["decay"] != "none":
            lam = np.log(np.asarray(c["g"], np.float64))
            lam = lam.reshape(1, T, 1) if c["decay"] == "diag" else lam.reshape(1, T)
        beta = None if c["update"] == "add" else np.asarray(c["beta"], np.float64).reshape(1, T)
        out, S = oracle.eager_tasks(np.array([[[c["s0"]]]], np.float64), a("q"), a("k"), a("v"),
                                    lam, beta, decay=c["decay"], update=c["update"],
                                    ckpts=[T], lib=lib)
        err = max(err, _rel(out.reshape(-1), c["o"]), _rel(S.reshape(-1), [c["s_T"]]))
    return err


ALL_PINS = [pin_additive_prefix_sum, pin_diag_decay_unrolled, pin_retention_parallel,
            pin_delta_matrix_form, pin_delta_invariants, pin_deferred_equals_eager,
            pin_scalar_golden]
