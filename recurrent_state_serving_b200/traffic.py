"""Algorithmic HBM bytes of the decode paths (the roofline numerator).

Counts the bytes a step must move at minimum, per head-step (one slot, one layer,
one value head), following the dense-state traffic model of the DeltaLog paper
(Background: eager materialisation reads and writes the dense d_k x d_v state every
token; Section 3: base + log replaces the write with compact appends, plus the log
replay reads and the periodic merge):

  eager            state read + write 8 d_k d_v                      + token I/O
  deferred append  state read 4 d_k d_v + c log entries read + 1 written + token I/O
  deferred merge   state read + write 8 d_k d_v + c log entries read     + token I/O
  standalone merge state read + write 8 d_k d_v + c log entries read

A log entry is a_i (4 d_k) + b_i (4 d_v) + Lambda_i (4 d_k for per-key decay, 4 for
scalar decay, 0 without decay).  In the compact layout a_i takes 2 d_k and, without
the delta rule, b_i takes 2 d_v (both are bf16 inputs, stored exactly).  Token I/O: q and k (shared by the n_heads/n_kheads
value heads of a group, so counted once per group), v, lambda (per step; a per-head
constant costs nothing per step), beta (delta rule) and the fp32 output.
"""
from __future__ import annotations

from .synth import Workload


def entry_bytes(wl: Workload, log_format: str = "fp32") -> int:
    lam = {"none": 0, "scalar": 4, "diag": 4 * wl.d_k}[wl.decay]
    if log_format == "compact":
        return 2 * wl.d_k + (4 if wl.update != "add" else 2) * wl.d_v + lam
    return 4 * wl.d_k + 4 * wl.d_v + lam


def token_bytes(wl: Workload, with_output: bool = True) -> float:
    esz = 2 if wl.in_dtype == "bf16" else 4
    group = wl.n_heads // wl.n_kheads
    b = 2 * wl.d_k * esz / group + wl.d_v * esz
    if wl.decay != "none" and not wl.lambda_const:
        b += 4 * wl.d_k if wl.decay == "diag" else 4
    if wl.update == "delta":
        b += 4
    if with_output:
        b += 4 * wl.d_v
    return b


def state_bytes(wl: Workload) -> int:
    return 4 * wl.d_k * wl.d_v


def eager_head_step(wl: Workload) -> float:
    return 2 * state_bytes(wl) + token_bytes(wl)


def deferred_head_step(wl: Workload, c: int, merge: bool, log_format: str = "fp32") -> float:
    """One decode step of one head whose log holds c live entries."""
    e = entry_bytes(wl, log_format)
    if merge:
        return 2 * state_bytes(wl) + c * e + token_bytes(wl)
    return state_bytes(wl) + c * e + e + token_bytes(wl)


def merge_head(wl: Workload, c: int, log_format: str = "fp32") -> float:
    return 2 * state_bytes(wl) + c * entry_bytes(wl, log_format)


def deferred_cycle_average(wl: Workload, log_format: str = "fp32") -> float:
    """Per head-step bytes averaged over one merge interval (c = 0 .. L-1, the last
    step of the interval being the merge step)."""
    L = wl.log_cap
    tot = sum(deferred_head_step(wl, c, merge=(c == L - 1), log_format=log_format) for c in range(L))
    return tot / L
