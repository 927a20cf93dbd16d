"""Drive a pool through decode steps for a synthetic workload.

A thin host-side loop over the C ABI: it allocates the pool (torch), writes the
prefill states, stages step inputs on the device and issues one library call per
layer and step.  All arithmetic happens in the library's kernels.

Slots: batch row b of the workload lives in pool slot ``slots[b]`` (a random
subset of a larger pool when ``n_slots > batch``, to exercise non-contiguous ids).
Staggering (per-slot log fill offsets) is realised by untimed pre-steps: before
the common steps, slot b takes ``offsets[b]`` decode steps with its own pre-step
inputs, so slots reach their merge steps at different times.

Slot groups: with ``n_groups = R > 1`` the pool holds R disjoint copies of the
batch's slots (group g uses ids ``g * per_group + slots``), each prefilled and
staggered the same way.  Stepping the groups in turn gives a working set R times
one step's, for timing a batch whose own state fits in L2 without an L2 flush.
"""
from __future__ import annotations

import numpy as np
import torch

from . import deltalog as dl
from . import synth


def _to_dev_input(a, in_dtype, device):
    if a is None:
        return None
    if in_dtype == "bf16" and a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


class DecodeRunner:
    def __init__(self, wl: synth.Workload, *, n_slots: int | None = None, slot_seed: int | None = None,
                 layers=None, mode: str = "deferred", update: str | None = None,
                 device: str = "cuda", tile_v: int = 0, n_groups: int = 1, log_format: str = "fp32",
                 replay: str = "per_tile"):
        if mode not in ("deferred", "eager"):
            raise ValueError(mode)
        self.wl = wl
        self.mode = mode
        self.update = update or wl.update
        self.device = torch.device(device)
        self.layers = list(range(wl.n_layers)) if layers is None else list(layers)
        n_slots = wl.batch if n_slots is None else n_slots
        if n_groups < 1:
            raise ValueError("n_groups must be >= 1")
        if slot_seed is None:
            ids = np.arange(wl.batch)
        else:
            ids = np.random.default_rng(slot_seed).permutation(n_slots)[:wl.batch]
        self.slot_ids = ids.astype(np.int32)
        self.group_slots = [torch.from_numpy((self.slot_ids + g * n_slots).astype(np.int32)).to(self.device)
                            for g in range(n_groups)]
        self.slots = self.group_slots[0]
        self.pool = dl.Pool(n_slots * n_groups, wl.n_layers, wl.n_heads, wl.d_k, wl.d_v, wl.log_cap,
                            decay=wl.decay, update=self.update, n_kheads=wl.n_kheads,
                            device=device, with_log=(mode == "deferred"), tile_v=tile_v,
                            log_format=log_format, replay=replay)
        self.offsets = synth.slot_offsets(wl)

    # -- set-up ----------------------------------------------------------------
    def load_initial_state(self):
        """Prefill: write each slot's initial state into the base, empty its log."""
        for layer in self.layers:
            S0 = torch.from_numpy(synth.initial_state(self.wl, layer)).to(self.device)
            for gs in self.group_slots:
                self.pool.state[gs.long(), layer] = S0
        for gs in self.group_slots:
            dl.dl_reset_slots(self.pool, gs)

    def device_inputs(self, inp: dict, rows=None) -> dict:
        if rows is not None:
            inp = synth.select_rows(self.wl, inp, rows)
        d = {k: _to_dev_input(v, self.wl.in_dtype if k in ("q", "k", "v") else "f32", self.device)
             for k, v in inp.items()}
        return d

    def gen_inputs(self, step: int, layer: int, prestep: bool = False) -> dict:
        return self.device_inputs(synth.step_inputs(self.wl, step, layer, prestep=prestep))

    # -- steps -----------------------------------------------------------------
    def call(self, layer: int, x: dict, slots=None, out=None, stream=None):
        """One library call for one layer (decode step or eager step)."""
        slots = self.slots if slots is None else slots
        fn = dl.dl_decode_step if self.mode == "deferred" else dl.dl_eager_step
        return fn(self.pool, layer, slots, x["q"], x["k"], x["v"], lam=x["lam"], beta=x["beta"],
                  out=out, lambda_per_head=self.wl.lambda_const, stream=stream)

    def run_presteps(self):
        """Staggering: slot b takes offsets[b] untimed decode steps first."""
        n = int(self.offsets.max()) if len(self.offsets) else 0
        for p in range(n):
            rows = np.nonzero(self.offsets > p)[0]
            sel = torch.from_numpy(rows).to(self.device)
            for layer in self.layers:
                x = self.device_inputs(synth.step_inputs(self.wl, p, layer, prestep=True), rows)
                for gs in self.group_slots:
                    self.call(layer, x, slots=gs[sel])

    def materialize(self, layer: int) -> torch.Tensor:
        if self.mode == "eager":
            return self.pool.state[self.slots.long(), layer].clone()
        return dl.dl_materialize(self.pool, layer, self.slots)

    def errors(self) -> int:
        return dl.dl_read_error(self.pool)
