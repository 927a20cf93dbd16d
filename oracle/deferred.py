"""fp64 deferred (base + log) decode of one head, written from the DeltaLog paper.

TEST INFRASTRUCTURE ONLY.  Used to pin the eager oracle (deferred with any merge
interval must equal eager) and to give the expected log contents.  It is never
the comparison for the GPU outputs themselves.

Follows the paper's notation (DeltaLog paper, "Append-merge decoding" and the
physical-state list that follows it):
  Sbar        dense base state produced by the most recent materialisation
  ellbar      cumulative log-decay applied since that materialisation
              (a scalar for head-wise scalar decay, a d_k vector for per-key decay)
  K_log, U_log, Lam_log   the bounded log: key factor a_i, value factor b_i and the
              log-decay snapshot taken when entry i was inserted
  live        the live-log length

The logical state (paper, recurrent-state traffic model) is
    S = D(ellbar) Sbar + sum_{i < live} D(ellbar - Lam_log[i]) K_log[i] U_log[i]^T,
with D(x) = Diag(exp(x)); the second term replays the deferred updates with
exactly the decay that accumulated after each was inserted.

A cycle of merge interval M has C = M - 1 append steps and one merge step; the
merge step decodes its token and then materialises the logical state into Sbar
and clears the log (ellbar = 0, live = 0).
"""
from __future__ import annotations

import numpy as np


class DeferredHead:
    def __init__(self, S0, rows: int, decay: str, update: str):
        """S0 [d_k, d_v]; rows = log capacity (= merge interval M)."""
        if decay not in ("none", "scalar", "diag"):
            raise ValueError(decay)
        if update not in ("add", "delta", "delta_undecayed"):
            raise ValueError(update)
        self.Sbar = np.array(S0, dtype=np.float64, copy=True)
        self.d_k, self.d_v = self.Sbar.shape
        self.rows = int(rows)
        self.decay = decay
        self.update = update
        self.ellbar = self._zero_decay()
        self.K_log, self.U_log, self.Lam_log = [], [], []

    # -- helpers ---------------------------------------------------------------
    def _zero_decay(self):
        return np.zeros(self.d_k) if self.decay == "diag" else 0.0

    def _as_decay(self, lam):
        if self.decay == "none":
            return 0.0
        if self.decay == "scalar":
            return float(lam)
        lam = np.asarray(lam, np.float64)
        assert lam.shape == (self.d_k,)
        return lam.copy()

    @staticmethod
    def _D(x, M):
        """Diag(exp(x)) M for a scalar or a per-row vector x."""
        e = np.exp(x)
        return (e[:, None] if np.ndim(e) else e) * M

    @property
    def live(self) -> int:
        return len(self.K_log)

    # -- the paper's logical state ---------------------------------------------
    def logical(self, ell=None):
        """D(ell) Sbar + sum_i D(ell - Lam_i) K_i U_i^T  (ell defaults to ellbar)."""
        ell = self.ellbar if ell is None else ell
        S = self._D(ell, self.Sbar)
        for a, b, Lam in zip(self.K_log, self.U_log, self.Lam_log):
            S = S + self._D(ell - Lam, np.outer(a, b))
        return S

    # -- operations -------------------------------------------------------------
    def append(self, k, v, lam=None, beta=None):
        """Record the compact update of one token; Sbar is left unchanged.
        Returns the value-side factor b that was logged."""
        if self.live >= self.rows:
            raise RuntimeError("log full")
        k = np.asarray(k, np.float64)
        v = np.asarray(v, np.float64)
        ell_t = self.ellbar + self._as_decay(lam)
        if self.update == "add":
            b = v.copy()
        else:
            # previous state, decayed by this step (delta) or as left by the last
            # step (delta_undecayed); both read off the logical state
            prev = self.logical(ell_t) if self.update == "delta" else self.logical()
            b = float(beta) * (v - prev.T @ k)
        self.K_log.append(k.copy())
        self.U_log.append(b)
        self.Lam_log.append(np.copy(ell_t) if np.ndim(ell_t) else float(ell_t))
        self.ellbar = ell_t
        return b

    def merge(self):
        """Materialise the logical state into Sbar and clear the log."""
        self.Sbar = self.logical()
        self.ellbar = self._zero_decay()
        self.K_log, self.U_log, self.Lam_log = [], [], []

    def decode(self, q, k, v, lam=None, beta=None, auto_merge: bool = True):
        """One decode step: append the token, read o_t = S_t^T q_t off the logical
        state, and merge when this step completes a merge interval."""
        if not auto_merge and self.live >= self.rows:
            raise RuntimeError("log full")
        if self.live >= self.rows:          # full log, auto-merge: no room to append
            self.rows += 1                  # the token is folded by the merge below
            try:
                self.append(k, v, lam, beta)
            finally:
                self.rows -= 1
        else:
            self.append(k, v, lam, beta)
        o = self.logical().T @ np.asarray(q, np.float64)
        if auto_merge and self.live >= self.rows:
            self.merge()
        return o
