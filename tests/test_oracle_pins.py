"""CPU tests: the fp64 oracle against what the mathematics fixes (no GPU)."""
import os
import shutil

import numpy as np
import pytest

import oracle
from oracle.deferred import DeferredHead
from tests import oracle_pins as P

TOL = 1e-12


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    assert pin() < TOL


# Mistakes a hand-written eager recurrence plausibly makes.  Each is planted in a
# private copy of the oracle; at least one pin must notice it.
MUTANTS = {
    "decay_dropped": ("Shat[(size_t)r * dv + c] = g[r] * S[(size_t)r * dv + c];",
                      "Shat[(size_t)r * dv + c] = S[(size_t)r * dv + c];"),
    "decay_sign_scalar": ("g[r] = exp(lam[t]);", "g[r] = exp(-lam[t]);"),
    "decay_sign_diag": ("g[r] = exp(lam[(size_t)t * dk + r]);",
                        "g[r] = exp(-lam[(size_t)t * dk + r]);"),
    "decay_step_off_by_one": ("g[r] = exp(lam[t]);", "g[r] = exp(lam[t > 0 ? t - 1 : 0]);"),
    "delta_readings_swapped": ("(dm->update == OR_UPDATE_DELTA) ? Shat : S",
                               "(dm->update == OR_UPDATE_DELTA) ? S : Shat"),
    "beta_dropped": ("b[c] = beta[t] * (vt[c] - u);", "b[c] = (vt[c] - u);"),
    "correction_sign": ("b[c] = beta[t] * (vt[c] - u);", "b[c] = beta[t] * (vt[c] + u);"),
    "correction_transposed": ("u += P[(size_t)r * dv + c] * kt[r];",
                              "u += P[(size_t)c * dk + r] * kt[r];"),
    "update_sign": ("= Shat[(size_t)r * dv + c] + kt[r] * b[c];",
                    "= Shat[(size_t)r * dv + c] - kt[r] * b[c];"),
    "update_uses_q": ("= Shat[(size_t)r * dv + c] + kt[r] * b[c];",
                      "= Shat[(size_t)r * dv + c] + qt[r] * b[c];"),
    "output_uses_k": ("o += S[(size_t)r * dv + c] * qt[r];", "o += S[(size_t)r * dv + c] * kt[r];"),
    "output_from_previous_state": ("o += S[(size_t)r * dv + c] * qt[r];",
                                   "o += Shat[(size_t)r * dv + c] * qt[r];"),
    "value_index": ("b[c] = vt[c];", "b[c] = vt[0];"),
    "checkpoint_off_by_one": ("if (ckpt_steps[j] == t + 1)", "if (ckpt_steps[j] == t)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {old}"
    mutant_src = tmp_path / "eager_mutant.c"
    mutant_src.write_text(src.replace(old, new, 1))
    lib_path = oracle.compile_c(str(mutant_src), str(tmp_path / "libmutant.so"))
    lib = oracle.load(lib_path)
    worst = 0.0
    for pin in P.ALL_PINS:
        try:
            worst = max(worst, pin(lib))
        except (AssertionError, RuntimeError, FloatingPointError, ValueError):
            worst = np.inf
        if worst > 1e-6:
            break
    assert worst > 1e-6, f"no pin caught mutant {name}"


def test_oracle_rejects_bad_arguments():
    import ctypes
    lib = oracle.load()
    buf = np.zeros(64)
    p = buf.ctypes.data_as(ctypes.c_void_p)
    ok = oracle._Dims(2, 2, 3, oracle.DECAY["none"], oracle.UPDATE["add"], 0)
    assert lib.oracle_eager_run(ctypes.byref(ok), 1, p, p, p, p, None, None, None, p, None, 1) == 0
    for dims in (oracle._Dims(2, 2, 3, oracle.DECAY["scalar"], oracle.UPDATE["add"], 0),  # no lambda
                 oracle._Dims(2, 2, 3, oracle.DECAY["none"], oracle.UPDATE["delta"], 0),  # no beta
                 oracle._Dims(0, 2, 3, 0, 0, 0), oracle._Dims(2, 2, 3, 7, 0, 0),
                 oracle._Dims(2, 2, 3, 0, 9, 0),
                 oracle._Dims(2, 2, 3, 0, 0, 1)):                                        # no ckpt buffer
        assert lib.oracle_eager_run(ctypes.byref(dims), 1, p, p, p, p, None, None, None, p,
                                    None, 1) == -1
    with pytest.raises(AssertionError):
        oracle.eager_tasks(np.zeros((1, 2, 2)), np.zeros((1, 3, 2)), np.zeros((1, 3, 2)),
                           np.zeros((1, 3, 2)), np.zeros((1, 2)), None, decay="scalar",
                           update="add")


def test_gva_head_mapping():
    """v-head h reads q/k of k-head h // (H / H_k); checked against per-head runs."""
    r = np.random.default_rng(5)
    T, B, H, Hk, dk, dv = 4, 2, 6, 3, 3, 2
    S0 = r.standard_normal((B, H, dk, dv))
    Q = r.standard_normal((T, B, Hk, dk))
    K = r.standard_normal((T, B, Hk, dk))
    V = r.standard_normal((T, B, H, dv))
    LAM = -0.1 * r.random((T, B, H, dk))
    BETA = r.random((T, B, H))
    O, S = oracle.eager_rollout(S0, Q, K, V, LAM, BETA, decay="diag", update="delta", ckpts=[T])
    for b in range(B):
        for h in range(H):
            g = h // (H // Hk)
            o1, s1 = oracle.eager_tasks(S0[b, h][None], Q[:, b, g][None], K[:, b, g][None],
                                        V[:, b, h][None], LAM[:, b, h][None], BETA[:, b, h][None],
                                        decay="diag", update="delta", ckpts=[T])
            np.testing.assert_array_equal(O[:, b, h], o1[0])
            np.testing.assert_array_equal(S[0, b, h], s1[0, 0])


def test_lambda_const_broadcast():
    r = np.random.default_rng(6)
    T, B, H, d = 5, 2, 3, 2
    S0 = r.standard_normal((B, H, d, d))
    Q, K = r.standard_normal((2, T, B, H, d))
    V = r.standard_normal((T, B, H, d))
    lam_h = -r.random(H)
    O1, _ = oracle.eager_rollout(S0, Q, K, V, lam_h, None, decay="scalar", update="add",
                                 lambda_const=True)
    O2, _ = oracle.eager_rollout(S0, Q, K, V, np.broadcast_to(lam_h, (T, B, H)), None,
                                 decay="scalar", update="add")
    np.testing.assert_array_equal(O1, O2)


def test_deferred_log_bookkeeping():
    """Merge interval M: C = M - 1 appends then one merge step, every cycle; the
    snapshot of entry i is the cumulative log-decay since the last merge."""
    r = np.random.default_rng(7)
    h = DeferredHead(r.standard_normal((3, 2)), 4, "diag", "delta")
    lives, since_merge = [], []
    for t in range(14):
        lam = -0.1 * r.random(3)
        h.decode(r.standard_normal(3), r.standard_normal(3), r.standard_normal(2), lam, 0.5)
        since_merge.append(lam)
        lives.append(h.live)
        if h.live == 0:
            since_merge = []
            assert np.all(h.ellbar == 0)
        else:
            np.testing.assert_allclose(h.Lam_log, np.cumsum(since_merge, axis=0), rtol=1e-15)
            np.testing.assert_array_equal(h.ellbar, h.Lam_log[-1])
    assert lives == [1, 2, 3, 0] * 3 + [1, 2]


def test_deferred_manual_append_merge_equals_eager():
    """dl_append/dl_merge flow: fill all L rows, merge, continue."""
    r = np.random.default_rng(8)
    dk, dv, T, L = 3, 4, 12, 4
    S0 = r.standard_normal((dk, dv))
    q, k = r.standard_normal((2, T, dk))
    v = r.standard_normal((T, dv))
    lam = -0.2 * r.random((T, dk))
    beta = r.random(T)
    out, S = oracle.eager_tasks(S0[None], q[None], k[None], v[None], lam[None], beta[None],
                                decay="diag", update="delta", ckpts=[T])
    h = DeferredHead(S0, L, "diag", "delta")
    for t in range(T):
        h.append(k[t], v[t], lam[t], beta[t])
        if h.live == L:
            h.merge()
    assert P._rel(h.logical(), S[0, 0]) < TOL
    with pytest.raises(RuntimeError):
        h2 = DeferredHead(S0, 2, "none", "add")
        for t in range(3):
            h2.append(k[t], v[t])
