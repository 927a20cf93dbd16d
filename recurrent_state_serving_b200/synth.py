"""Seeded synthetic inputs for the recurrent-state decode workloads.

This module is shared by the CUDA path's harness (tests, benchmark) and by the
CPU oracle's harness.  It draws inputs only: it holds none of the decode
method's arithmetic.  Everything is deterministic in (seed, tensor tag, step,
layer): each (tag, step, layer) triple owns one Philox-4x64 stream (numpy's
counter-based generator), so any single step/layer of a large workload can be
regenerated on its own, for example to check a sampled head of a full-size run.

16-bit inputs are rounded to bfloat16 with round-to-nearest-even from their
fp32 value and handed out as raw uint16 bit patterns; both sides read the same
bits (the GPU as bf16, the oracle upcast exactly to fp64).

Workload shapes follow the kernel sweeps of the DeltaLog paper ("DeltaLog:
Deferred Materialization of Recurrent States for Linear Attention Decoding",
evaluation section: H=32, d=128, fp32 state, B in {64..512}, merge interval
M in {2..64}) and the GDN batch-1 shape of "A Persistent-State Dataflow
Accelerator for Memory-Bound Linear Attention Decode on FPGA" (Table II:
h_v=32, d=128, FP32).
"""
from __future__ import annotations

from dataclasses import dataclass, replace
import math

import numpy as np

# Stream tags (one Philox key per tag/step/layer).
_TAG_Q, _TAG_K, _TAG_V, _TAG_LAM, _TAG_BETA, _TAG_S0, _TAG_OFFS = 1, 2, 3, 4, 5, 6, 7
_PRESTEP = 1 << 8        # tag bit for the untimed staggering pre-steps


@dataclass(frozen=True)
class Workload:
    """One decode workload.  Names follow the paper's notation:
    H v-heads (H_k k-heads for grouped value attention), d_k x d_v state per
    head, merge interval / log capacity L, decay granularity and update rule."""
    name: str
    n_layers: int
    batch: int
    n_heads: int
    n_kheads: int
    d_k: int
    d_v: int
    in_dtype: str          # 'f32' or 'bf16' for q, k, v
    decay: str             # 'none' | 'scalar' | 'diag'
    lambda_const: bool     # True: one log-decay per head, fixed over steps/slots
    update: str            # 'add' (b = v) | 'delta' (b = beta (v - S^T k))
    steps: int
    log_cap: int           # L: merge every L steps
    seed: int
    qkv_std: float
    init_std: float        # 0 means a zero initial state
    k_l2norm: bool
    lam_mean: float        # lambda = logsigmoid(x), x ~ N(lam_mean, 1)
    staggered: bool        # per-slot random log fill offsets in [0, L)

    @property
    def units_per_step(self) -> int:
        """Head-steps in one decode step of the whole batch over all layers."""
        return self.batch * self.n_heads * self.n_layers

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads: tiny no-decay linear attention; GLA/RWKV6-style diagonal
# decay; GDN with grouped value attention at batch 1; KDA-style per-key decay with
# the delta rule; RetNet scalar decay with staggered merges.
TINY_LA = Workload("tiny_la", 1, 1, 2, 2, 16, 16, "f32", "none", False, "add",
                   32, 4, 1000, 1.0 / math.sqrt(16), 0.0, False, 0.0, False)
GLA_DIAG = Workload("gla_rwkv6_diag", 1, 64, 16, 16, 128, 128, "bf16", "diag", False,
                    "add", 256, 8, 1001, 1.0 / math.sqrt(128), 0.02, False, 4.0, False)
GDN_GVA = Workload("gdn_gva", 1, 1, 32, 16, 128, 128, "bf16", "scalar", False, "delta",
                   128, 16, 1002, 1.0 / math.sqrt(128), 0.0, True, 3.0, False)
KDA = Workload("kda_diag_delta", 24, 256, 32, 32, 128, 128, "bf16", "diag", False,
               "delta", 64, 16, 1003, 1.0 / math.sqrt(128), 0.02, True, 4.0, False)
RETNET = Workload("retnet_scalar", 8, 256, 32, 32, 128, 128, "bf16", "scalar", True,
                  "add", 128, 32, 1004, 1.0 / math.sqrt(128), 0.02, False, 0.0, True)

WORKLOADS = {w.name: w for w in (TINY_LA, GLA_DIAG, GDN_GVA, KDA, RETNET)}
GLA_LOG_CAPS = (4, 8, 16, 32)
RETNET_BATCHES = (1, 16, 64, 256, 1024)


# ----------------------------------------------------------------------------
# bit-level helpers
# ----------------------------------------------------------------------------
def to_bf16_bits(x) -> np.ndarray:
    """Round to bfloat16 (nearest-even from the fp32 value); returns uint16 bits."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, tag: int, step: int, layer: int) -> np.random.Generator:
    if not (0 <= step < (1 << 24) and 0 <= layer < (1 << 16) and 0 <= tag < (1 << 20)):
        raise ValueError("stream coordinates out of range")
    key = np.array([seed, (tag << 40) | (step << 16) | layer], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def _logsigmoid(x):
    # log(sigmoid(x)) = -log1p(exp(-x)), stable form for both signs
    return np.where(x >= 0, -np.log1p(np.exp(-np.abs(x))), x - np.log1p(np.exp(-np.abs(x))))


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _as_input(x64, in_dtype):
    return to_bf16_bits(x64) if in_dtype == "bf16" else np.asarray(x64, np.float32)


def input_to_f64(x, in_dtype) -> np.ndarray:
    """Exact upcast of a generated q/k/v array to float64."""
    if in_dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, np.float32).astype(np.float64)


def retnet_log_decay(n_heads: int) -> np.ndarray:
    """lambda_h = log(1 - 2^(-5 - 5h/32)) for h = 0..H-1 (fp32)."""
    h = np.arange(n_heads, dtype=np.float64)
    return np.log1p(-np.exp2(-5.0 - 5.0 * h / 32.0)).astype(np.float32)


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------
def step_inputs(wl: Workload, step: int, layer: int, prestep: bool = False) -> dict:
    """Inputs of one decode step for all wl.batch rows of one layer.

    Returns a dict with
      q, k : [B, H_k, d_k]  (uint16 bf16 bits or float32)
      v    : [B, H, d_v]
      lam  : None | [B, H] (scalar) | [B, H, d_k] (diag) | [H] / [H, d_k] if lambda_const
      beta : None | [B, H] float32
    """
    B, H, Hk, dk, dv = wl.batch, wl.n_heads, wl.n_kheads, wl.d_k, wl.d_v
    t = _PRESTEP if prestep else 0
    s = wl.qkv_std
    q = _rng(wl.seed, _TAG_Q | t, step, layer).standard_normal((B, Hk, dk)) * s
    k = _rng(wl.seed, _TAG_K | t, step, layer).standard_normal((B, Hk, dk)) * s
    if wl.k_l2norm:
        k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    v = _rng(wl.seed, _TAG_V | t, step, layer).standard_normal((B, H, dv)) * s
    out = {"q": _as_input(q, wl.in_dtype), "k": _as_input(k, wl.in_dtype),
           "v": _as_input(v, wl.in_dtype), "lam": None, "beta": None}
    if wl.decay != "none":
        if wl.lambda_const:
            lam = retnet_log_decay(H)
            if wl.decay == "diag":
                lam = np.repeat(lam[:, None], dk, axis=1)
            out["lam"] = np.ascontiguousarray(lam, dtype=np.float32)
        else:
            shape = (B, H) if wl.decay == "scalar" else (B, H, dk)
            x = _rng(wl.seed, _TAG_LAM | t, step, layer).standard_normal(shape) + wl.lam_mean
            out["lam"] = _logsigmoid(x).astype(np.float32)
    if wl.update == "delta":
        x = _rng(wl.seed, _TAG_BETA | t, step, layer).standard_normal((B, H))
        out["beta"] = _sigmoid(x).astype(np.float32)
    return out


def initial_state(wl: Workload, layer: int) -> np.ndarray:
    """Initial (prefill) state [B, H, d_k, d_v] float32; N(0, init_std^2) or zero."""
    shape = (wl.batch, wl.n_heads, wl.d_k, wl.d_v)
    if wl.init_std == 0.0:
        return np.zeros(shape, np.float32)
    g = _rng(wl.seed, _TAG_S0, 0, layer)
    return (g.standard_normal(shape) * wl.init_std).astype(np.float32)


def slot_offsets(wl: Workload) -> np.ndarray:
    """Per-slot log fill offset in [0, L): the number of untimed pre-steps a slot
    takes before the common steps, so that merges are staggered across slots."""
    if not wl.staggered:
        return np.zeros(wl.batch, np.int64)
    return _rng(wl.seed, _TAG_OFFS, 0, 0).integers(0, wl.log_cap, size=wl.batch)


def select_rows(wl: Workload, inputs: dict, rows) -> dict:
    """Restrict a step_inputs() dict to a subset of batch rows."""
    out = {}
    for key, val in inputs.items():
        if val is None or (key == "lam" and wl.lambda_const):
            out[key] = val
        else:
            out[key] = np.ascontiguousarray(val[rows])
    return out
