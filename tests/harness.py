"""Test harness: run a workload through the CUDA path and through the fp64 oracle
on the same seeded inputs, and compare.  Test infrastructure only."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from recurrent_state_serving_b200 import synth
from recurrent_state_serving_b200.runner import DecodeRunner

# Tolerances.  The accuracy bound of this path: relative L2 error of each step's whole
# output tensor (and of each checkpointed state) against the fp64 oracle <= 1e-4.  Per
# element we also require |gpu - ref| <= 1e-3 * RMS(ref of that step): the fp32
# path accumulates d_k-term dot products (error ~ sqrt(d_k) * 2^-24 relative), so a
# single element 10x above the average allowed error already indicates a bug.
REL_L2 = 1e-4
ELEM_RMS = 1e-3
# GPU deferred vs GPU eager (both fp32): relative L2 per step <= 1e-5.
REL_L2_GPU = 1e-5


def rel_l2(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / d) if d > 0 else float(np.linalg.norm(x))


def check_steps(gpu, ref, tol=REL_L2, elem=ELEM_RMS, what="output"):
    """gpu, ref: [T, ...].  Returns the worst per-step relative L2 error."""
    worst = 0.0
    for t in range(ref.shape[0]):
        e = rel_l2(gpu[t], ref[t])
        worst = max(worst, e)
        assert e <= tol, f"{what} step {t}: rel-L2 {e:.3e} > {tol:.0e}"
        if elem is not None:
            rms = np.sqrt(np.mean(np.asarray(ref[t], np.float64) ** 2))
            dmax = np.max(np.abs(np.asarray(gpu[t], np.float64) - ref[t]))
            assert dmax <= elem * rms, f"{what} step {t}: max |err| {dmax:.3e} > {elem} * RMS {rms:.3e}"
    return worst


def stack_inputs(wl: synth.Workload, seq: list, rows) -> dict:
    """seq: list of step_inputs() dicts (full batch).  Returns float64 arrays over the
    given rows: Q, K [T, R, H_k, d_k], V [T, R, H, d_v], LAM, BETA."""
    f = lambda x: synth.input_to_f64(x, wl.in_dtype)
    out = {"Q": np.stack([f(x["q"][rows]) for x in seq]),
           "K": np.stack([f(x["k"][rows]) for x in seq]),
           "V": np.stack([f(x["v"][rows]) for x in seq]),
           "LAM": None, "BETA": None}
    if wl.decay != "none":
        if wl.lambda_const:
            out["LAM"] = seq[0]["lam"].astype(np.float64)
        else:
            out["LAM"] = np.stack([x["lam"][rows].astype(np.float64) for x in seq])
    if wl.update == "delta":
        out["BETA"] = np.stack([x["beta"][rows].astype(np.float64) for x in seq])
    return out


def oracle_reference(wl: synth.Workload, layer: int, T: int, rows=None, ckpts=(), update=None,
                     main_inputs=None, main_selected=False):
    """Eager fp64 reference for the rows' main steps 0..T-1 (after their staggering
    pre-steps).  ckpts count main steps (0 = after the pre-steps).  main_inputs: the
    main steps' step_inputs() dicts (full batch, or only `rows` when main_selected).
    Returns O [T, R, H, d_v], S [len(ckpts), R, H, d_k, d_v]."""
    rows = np.arange(wl.batch) if rows is None else np.asarray(rows)
    update = update or wl.update
    offs = synth.slot_offsets(wl)[rows]
    S0 = synth.initial_state(wl, layer)[rows].astype(np.float64)
    sel = lambda x: synth.select_rows(wl, x, rows)
    if main_inputs is None:
        main = [sel(synth.step_inputs(wl, t, layer)) for t in range(T)]
    else:
        main = list(main_inputs) if main_selected else [sel(x) for x in main_inputs]
    pre = [sel(synth.step_inputs(wl, p, layer, prestep=True)) for p in range(int(offs.max()))]
    R = len(rows)
    O = np.zeros((T, R, wl.n_heads, wl.d_v))
    S = np.zeros((len(ckpts), R, wl.n_heads, wl.d_k, wl.d_v))
    for o in np.unique(offs):
        idx = np.nonzero(offs == o)[0]
        x = stack_inputs(wl, pre[:o] + main, idx)
        Oo, So = oracle.eager_rollout(S0[idx], x["Q"], x["K"], x["V"], x["LAM"], x["BETA"],
                                      decay=wl.decay, update=update,
                                      lambda_const=wl.lambda_const,
                                      ckpts=[int(o) + c for c in ckpts])
        O[:, idx] = Oo[o:]
        S[:, idx] = So
    return O, S


def gpu_rollout(runner: DecodeRunner, T: int, ckpts=(), layers=None, keep_inputs=False, state_rows=None,
                out_rows=None):
    """Run T common steps (after set-up and pre-steps) on the GPU.
    Returns ({layer: O [T, B, H, d_v]}, {layer: S [len(ckpts), B, H, d_k, d_v]},
    {layer: [host inputs per step]}).  state_rows / out_rows: keep only these batch
    rows of the checkpointed states / outputs (the device still runs every row); with
    out_rows the kept inputs hold only those rows too (oracle_reference(...,
    main_selected=True))."""
    layers = runner.layers if layers is None else layers
    wl = runner.wl
    runner.load_initial_state()
    runner.run_presteps()
    outs = {l: [] for l in layers}
    states = {l: [] for l in layers}
    kept = {l: [] for l in layers}
    sel = None if state_rows is None else torch.as_tensor(np.asarray(state_rows), device=runner.device)
    osel = None if out_rows is None else torch.as_tensor(np.asarray(out_rows), device=runner.device)

    def snap(l):
        S = runner.materialize(l)
        if sel is not None:
            S = S.index_select(0, sel)
        return S.double().cpu().numpy()
    for l in layers:
        if 0 in ckpts:
            states[l].append(snap(l))
    for t in range(T):
        for l in layers:
            host = synth.step_inputs(wl, t, l)
            if keep_inputs:
                kept[l].append(host if out_rows is None else synth.select_rows(wl, host, np.asarray(out_rows)))
            o = runner.call(l, runner.device_inputs(host))
            if osel is not None:
                o = o.index_select(0, osel)
            outs[l].append(o.double().cpu().numpy())
            if t + 1 in ckpts:
                states[l].append(snap(l))
    torch.cuda.synchronize()
    return ({l: np.stack(v) for l, v in outs.items()},
            {l: (np.stack(v) if v else None) for l, v in states.items()}, kept)


def log_entries_f64(pool) -> np.ndarray:
    """The pool's log ring as float64 [slot, layer, head, L, 2 d_k + d_v] rows
    [a | b | Lambda], whatever its layout (test-side decoding of the compact layout:
    bf16 a, bf16 b without the delta rule, Lambda fp32 x d_k / x 4 / none)."""
    raw = pool.log.detach().cpu().contiguous()
    dk, dv = pool.d_k, pool.d_v
    if pool.log_format == "fp32":
        return raw.double().numpy()
    words = raw.view(torch.int32).numpy()
    lead = words.shape[:-1]
    out = np.zeros(lead + (2 * dk + dv,), np.float64)

    def bf16(w):   # packed pairs of bf16 in 32-bit words -> float64
        h = w.view(np.uint32)
        lo = (h & np.uint32(0xFFFF)).astype(np.uint32) << np.uint32(16)
        hi = h & np.uint32(0xFFFF0000)
        return np.stack([lo.view(np.float32), hi.view(np.float32)], axis=-1).reshape(w.shape[:-1] + (-1,)).astype(np.float64)

    def f32(w):
        return w.view(np.float32).astype(np.float64)

    out[..., :dk] = bf16(words[..., :dk // 2])
    boff = dk // 2
    if pool.update == "add":
        out[..., dk:dk + dv] = bf16(words[..., boff:boff + dv // 2])
        loff = boff + dv // 2
    else:
        out[..., dk:dk + dv] = f32(words[..., boff:boff + dv])
        loff = boff + dv
    if pool.decay == "diag":
        out[..., dk + dv:] = f32(words[..., loff:loff + dk])
    elif pool.decay == "scalar":
        out[..., dk + dv] = f32(words[..., loff])
    return out
