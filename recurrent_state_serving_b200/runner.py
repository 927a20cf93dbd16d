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
batch's slots (group g uses ids ``g * per_group + slots``), each prefilled the
same way and staggered by its own row of ``offsets`` (the workload's offsets for
every group unless given).  Stepping the groups in turn gives a working set R
times one step's, for timing a batch whose own state fits in L2 without an L2
flush.
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
                 replay: str = "per_tile", offsets=None, merge="capacity"):
        if mode not in ("deferred", "eager"):
            raise ValueError(mode)
        self.wl = wl
        self.mode = mode
        self.merge = merge   # dl_decode_step's merge policy: 'capacity', 'adaptive' or 'none'
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
        # per-group staggering offsets [n_groups, batch]
        if offsets is None:
            self.group_offsets = np.tile(self.offsets, (n_groups, 1))
        else:
            go = np.asarray(offsets, dtype=np.int64)
            if go.shape != (n_groups, wl.batch) or (go < 0).any():
                raise ValueError("offsets must be non-negative with shape [n_groups, batch]")
            self.group_offsets = go
            self.offsets = go[0]

    # -- set-up ----------------------------------------------------------------
    def load_initial_state(self, on_device: bool = False):
        """Prefill: write each slot's initial state into the base, empty its log.

        on_device: draw N(0, init_std^2) states with torch's seeded device generator
        instead of synth.initial_state (much faster for multi-GB pools; the values
        then differ from the oracle's, so this is for timing only)."""
        for layer in self.layers:
            if on_device:
                shape = (self.wl.batch, self.wl.n_heads, self.wl.d_k, self.wl.d_v)
                if self.wl.init_std == 0.0:
                    S0 = torch.zeros(shape, dtype=torch.float32, device=self.device)
                else:
                    g = torch.Generator(device=self.device)
                    g.manual_seed(self.wl.seed * 1000 + layer)
                    S0 = torch.randn(shape, generator=g, dtype=torch.float32, device=self.device)
                    S0.mul_(self.wl.init_std)
            else:
                S0 = torch.from_numpy(synth.initial_state(self.wl, layer)).to(self.device)
            for gs in self.group_slots:
                self.pool.state[gs.long(), layer] = S0
            del S0
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
    def call(self, layer: int, x: dict, slots=None, out=None, stream=None, merge=None):
        """One library call for one layer (decode step or eager step); merge overrides
        the runner's merge policy for this call."""
        slots = self.slots if slots is None else slots
        if self.mode == "eager":
            return dl.dl_eager_step(self.pool, layer, slots, x["q"], x["k"], x["v"], lam=x["lam"],
                                    beta=x["beta"], out=out, lambda_per_head=self.wl.lambda_const,
                                    stream=stream)
        return dl.dl_decode_step(self.pool, layer, slots, x["q"], x["k"], x["v"], lam=x["lam"],
                                 beta=x["beta"], out=out, lambda_per_head=self.wl.lambda_const,
                                 auto_merge=self.merge if merge is None else merge, stream=stream)

    def run_presteps(self, inputs=None):
        """Staggering: slot b of group g takes group_offsets[g, b] untimed decode steps
        first.  inputs(p, layer) -> device inputs of the whole batch for pre-step p
        (default: the workload's own seeded pre-step inputs).  The pre-steps run on
        sub-batches with the at-capacity merge policy whatever the runner's policy is:
        the adaptive one would merge a small sub-batch on every step and undo the
        staggering."""
        go = self.group_offsets
        n = int(go.max()) if go.size else 0
        for p in range(n):
            for layer in self.layers:
                if inputs is None:
                    xh = synth.step_inputs(self.wl, p, layer, prestep=True)
                x_all = None
                for g, gs in enumerate(self.group_slots):
                    rows = np.nonzero(go[g] > p)[0]
                    if len(rows) == 0:
                        continue
                    if inputs is None:
                        x = self.device_inputs(xh, rows)
                    else:
                        if x_all is None:
                            x_all = inputs(p, layer)
                        x = self.select_device_rows(x_all, rows)
                    sel = torch.from_numpy(rows).to(self.device)
                    self.call(layer, x, slots=gs[sel], merge="capacity")

    def select_device_rows(self, x: dict, rows) -> dict:
        """Rows of a device input dict (a per-head constant lambda is kept whole)."""
        idx = torch.as_tensor(np.asarray(rows), device=self.device, dtype=torch.long)
        out = {}
        for k, v in x.items():
            if v is None or (k == "lam" and self.wl.lambda_const):
                out[k] = v
            else:
                out[k] = v.index_select(0, idx).contiguous()
        return out

    def materialize(self, layer: int) -> torch.Tensor:
        if self.mode == "eager":
            return self.pool.state[self.slots.long(), layer].clone()
        return dl.dl_materialize(self.pool, layer, self.slots)

    def errors(self) -> int:
        return dl.dl_read_error(self.pool)
