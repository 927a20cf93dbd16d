"""Choice of the merge interval L (the log capacity) per operator.

The DeltaLog paper (Evaluation, the merge-interval study of Figure 10) sweeps the
merge interval for each operator and keeps the best one.  The amortised step time is
U-shaped in L.  A small L writes the dense state back often. A large L replays a
longer log on every append.  The best interval differs between operators, because
their log entries differ in size (per-key decay carries a d_k-float Lambda, scalar
decay one float, the compact layout half-width a and b).

Two selectors:

* ``modelled_log_cap`` minimises the algorithmic HBM bytes per head-step, averaged
  over one interval (``traffic.deferred_cycle_average``), over a candidate list.
  With S = 4 d_k d_v state bytes and e bytes per log entry, the interval-dependent
  part of that average is (S - e) / L + e L / 2, whose real minimiser is
  sqrt(2 (S - e) / e).  This is the answer for an HBM-bound launch (many heads per SM).
* ``select_log_cap`` picks from measured rates per candidate, as the paper does.  A
  launch with few heads per SM is latency-bound, and there a smaller L (or L = 1,
  which is the eager recurrence) can win although it moves more bytes.

Ties go to the smaller L: it holds less log memory per slot.
"""
from __future__ import annotations

import math

from . import synth, traffic
from .synth import Workload

DEFAULT_CANDIDATES = (1, 2, 4, 8, 16, 32, 64)


def cycle_bytes(wl: Workload, log_cap: int, log_format: str = "fp32") -> float:
    """Algorithmic bytes per head-step averaged over one interval of length log_cap."""
    if log_cap < 1:
        raise ValueError("log_cap must be >= 1")
    return traffic.deferred_cycle_average(wl.with_(log_cap=log_cap), log_format)


def modelled_log_cap(wl: Workload, candidates=DEFAULT_CANDIDATES, log_format: str = "fp32") -> int:
    """The candidate with the fewest algorithmic bytes per head-step (smallest on ties)."""
    cands = sorted(set(int(c) for c in candidates))
    if not cands or cands[0] < 1:
        raise ValueError("candidates must be positive integers")
    return min(cands, key=lambda L: (cycle_bytes(wl, L, log_format), L))


def auto_log_cap(d_k: int, d_v: int, decay: str, update: str, log_format: str = "fp32",
                 candidates=DEFAULT_CANDIDATES) -> int:
    """The modelled interval for an operator given by its shape alone (the per-step
    token bytes do not depend on L, so batch, heads and input type do not matter)."""
    wl = synth.GLA_DIAG.with_(name="operator", d_k=d_k, d_v=d_v, decay=decay, update=update)
    return modelled_log_cap(wl, candidates, log_format)


def continuous_optimum(wl: Workload, log_format: str = "fp32") -> float:
    """Real minimiser of the byte model over L > 0: sqrt(2 (S - e) / e)."""
    S = traffic.state_bytes(wl)
    e = traffic.entry_bytes(wl, log_format)
    if e <= 0 or S <= e:
        raise ValueError("the byte model has no interior minimum for this shape")
    return math.sqrt(2.0 * (S - e) / e)


def select_log_cap(measured: dict, higher_is_better: bool = True) -> int:
    """The fastest interval from measured results {L: rate or time}.

    ``measured`` maps each candidate L to a throughput (``higher_is_better``) or a time
    per step.  Candidates measured as None or NaN are skipped.
    """
    pts = []
    for L, v in measured.items():
        if v is None or (isinstance(v, float) and math.isnan(v)):
            continue
        if int(L) < 1:
            raise ValueError("log_cap must be >= 1")
        pts.append((int(L), float(v)))
    if not pts:
        raise ValueError("no measured candidate")
    sign = -1.0 if higher_is_better else 1.0
    return min(pts, key=lambda p: (sign * p[1], p[0]))[0]


def select_from_bench_lines(lines) -> dict:
    """Best interval per operator configuration from bench JSON lines.

    Each line is one ``bench.py --log-cap L`` run (a JSON object, or its text).  Lines
    are grouped by everything in their ``config`` that does not depend on L (workload
    shape, decay, update rule, log layout, batch, GPU count); reference-arm lines and
    lines without a value are skipped.  Returns {group key: (best L, {L: value})}, the
    key being the workload name without its ``_L<n>`` part plus the log layout."""
    import json
    import re

    groups: dict = {}
    for ln in lines:
        d = json.loads(ln) if isinstance(ln, str) else ln
        if not isinstance(d, dict) or d.get("impl") == "reference" or d.get("value") is None:
            continue
        cfg = d.get("config", {})
        if "log_cap" not in cfg or "workload" not in cfg:
            continue
        L = int(cfg["log_cap"])
        base = re.sub(r"_L\d+", "", cfg["workload"])
        key = (base, cfg.get("log_format", "fp32"), int(d.get("n_gpus", 1)))
        better = d.get("higher_is_better", True)
        g = groups.setdefault(key, ({}, better))
        g[0][L] = float(d["value"])
    return {f"{b} [{fmt}, {n} GPU]": (select_log_cap(vals, better), vals)
            for (b, fmt, n), (vals, better) in groups.items()}


def sweep_table(wl: Workload, candidates=DEFAULT_CANDIDATES, log_format: str = "fp32"):
    """(L, bytes per head-step, bytes relative to the eager step) for each candidate."""
    eager = traffic.eager_head_step(wl)
    rows = []
    for L in sorted(set(int(c) for c in candidates)):
        b = cycle_bytes(wl, L, log_format)
        rows.append((L, b, b / eager))
    return rows


def main(argv=None):
    import argparse

    ap = argparse.ArgumentParser(description="Merge interval per operator from the byte model")
    ap.add_argument("--workload", default="gla_rwkv6_diag", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--log-format", default="fp32", choices=["fp32", "compact"])
    ap.add_argument("--candidates", default=",".join(str(c) for c in DEFAULT_CANDIDATES))
    ap.add_argument("--from-bench", default=None,
                    help="file of bench.py JSON lines (one per --log-cap run): print the measured pick")
    a = ap.parse_args(argv)
    if a.from_bench:
        with open(a.from_bench) as f:
            lines = [ln for ln in f if ln.strip().startswith("{")]
        for key, (best, vals) in sorted(select_from_bench_lines(lines).items()):
            rates = ", ".join(f"L={L}: {v:.4g}" for L, v in sorted(vals.items()))
            print(f"{key}: measured best L = {best} ({rates})")
        return
    wl = synth.WORKLOADS[a.workload]
    cands = [int(x) for x in a.candidates.split(",") if x]
    for L, b, r in sweep_table(wl, cands, a.log_format):
        print(f"L={L:3d}  {b / 1024:8.2f} KiB per head-step  {r:6.3f} of eager")
    print(f"modelled best L = {modelled_log_cap(wl, cands, a.log_format)} "
          f"(real optimum {continuous_optimum(wl, a.log_format):.2f})")


if __name__ == "__main__":
    main()
