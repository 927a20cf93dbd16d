"""Serving loop around the decode step: slot admission, retirement, graph replay.

The DeltaLog paper's serving integration (its CUDA-graph and allocator passages)
keeps, per request slot, the dense state from prefill plus a bounded log, gives a
fresh request a slot whose log metadata is reset, and captures separate append and
merge CUDA graphs per decode-batch descriptor.  Here one kernel serves both phases:
each slot takes its merge step on its own L-th step inside the same launch, so one
graph per batch size covers every mix of append and merge slots, and requests
admitted at different times merge at different steps without any queueing.

``DecodeServer`` owns a pool (the library allocates nothing; torch holds the
buffers), a host-side free list of slots, and fixed device buffers for one step's
inputs at a maximum batch size.  A decode step copies the active rows' inputs into
those buffers and replays the CUDA graph captured for that batch size (all layers,
one ``dl_decode_step`` per layer).  All arithmetic is in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import deltalog as dl
from . import tuning


class SlotAllocator:
    """Free list of pool slots (host side).  Lowest free id first, so a retired
    slot is the next one handed out."""

    def __init__(self, n_slots: int):
        if n_slots <= 0:
            raise ValueError("n_slots must be positive")
        self.n_slots = n_slots
        self._free = list(range(n_slots - 1, -1, -1))
        self._used = set()

    def alloc(self) -> int:
        if not self._free:
            raise RuntimeError("no free slot")
        s = self._free.pop()
        self._used.add(s)
        return s

    def free(self, s: int):
        if s not in self._used:
            raise ValueError(f"slot {s} is not allocated")
        self._used.remove(s)
        self._free.append(s)
        self._free.sort(reverse=True)

    @property
    def n_free(self) -> int:
        return len(self._free)

    @property
    def used(self):
        return sorted(self._used)


@dataclass
class Request:
    rid: int
    slot: int
    steps: int = 0              # decode steps taken


class DecodeServer:
    """Batched decode over a slot pool with admission and retirement.

    Inputs of a step are given per layer as dicts of device tensors with one row per
    active request, in the order of ``active`` (q, k: [B, H_k, d_k]; v: [B, H, d_v];
    lam: [B, H] / [B, H, d_k] or per-head constants; beta: [B, H]).

    ``log_cap="auto"`` takes the merge interval with the fewest modelled HBM bytes per
    head-step for this operator's shape, decay, update rule and log layout
    (``tuning.auto_log_cap``), which is the right choice when the batch fills the GPU.

    ``merge`` is the library's merge policy: "capacity" (each slot merges on its L-th
    step) or "adaptive" (as "capacity", but a batch too small to fill the GPU merges
    every slot on every step, which is faster there; dl_merge_policy tells which).
    """

    def __init__(self, *, n_slots, n_layers, n_heads, d_k, d_v, log_cap, decay="none",
                 update="add", n_kheads=None, in_dtype=torch.bfloat16, lambda_per_head=False,
                 log_format="fp32", tile_v=0, max_batch=None, device="cuda", use_graphs=True,
                 merge="capacity"):
        if log_cap == "auto":
            log_cap = tuning.auto_log_cap(d_k, d_v, decay, update, log_format)
        self.log_cap = int(log_cap)
        if merge not in ("capacity", "adaptive"):
            raise ValueError("merge must be 'capacity' or 'adaptive'")
        self.merge = merge
        self.pool = dl.Pool(n_slots, n_layers, n_heads, d_k, d_v, self.log_cap, decay=decay,
                            update=update, n_kheads=n_kheads, device=device, log_format=log_format,
                            tile_v=tile_v)
        self.alloc = SlotAllocator(n_slots)
        self.n_layers, self.H = n_layers, n_heads
        self.Hk = n_heads if n_kheads is None else n_kheads
        self.d_k, self.d_v, self.decay, self.update = d_k, d_v, decay, update
        self.lambda_per_head = lambda_per_head
        self.max_batch = n_slots if max_batch is None else max_batch
        self.device = torch.device(device)
        self.use_graphs = use_graphs
        self.requests: dict[int, Request] = {}
        self.active: list[int] = []          # request ids, row order of the batch
        self._next_rid = 0
        B, dev = self.max_batch, self.device
        # fixed per-step buffers (graph operands)
        self.slots_buf = torch.zeros(B, dtype=torch.int32, device=dev)
        self.bufs = []
        for _ in range(n_layers):
            b = {"q": torch.zeros(B, self.Hk, d_k, dtype=in_dtype, device=dev),
                 "k": torch.zeros(B, self.Hk, d_k, dtype=in_dtype, device=dev),
                 "v": torch.zeros(B, n_heads, d_v, dtype=in_dtype, device=dev),
                 "lam": None, "beta": None,
                 "out": torch.zeros(B, n_heads, d_v, dtype=torch.float32, device=dev)}
            if decay != "none" and not lambda_per_head:
                shape = (B, n_heads) if decay == "scalar" else (B, n_heads, d_k)
                b["lam"] = torch.zeros(shape, dtype=torch.float32, device=dev)
            if update != "add":
                b["beta"] = torch.zeros(B, n_heads, dtype=torch.float32, device=dev)
            self.bufs.append(b)
        self.lam_const = [None] * n_layers   # per-head constants, set by set_lambda_per_head
        self._graphs: dict[int, torch.cuda.CUDAGraph] = {}
        self._prepared: dict[int, list] = {}

    # -- requests ------------------------------------------------------------------
    def admit(self, prefill_state: torch.Tensor) -> int:
        """A fresh request: its prefill state [n_layers, H, d_k, d_v] fp32 becomes the
        dense base of a free slot, whose log is reset.  Returns the request id."""
        if len(self.active) >= self.max_batch:
            raise RuntimeError("batch is full")
        want = (self.n_layers, self.H, self.d_k, self.d_v)
        if tuple(prefill_state.shape) != want:
            raise ValueError(f"prefill state must be {list(want)}")
        s = self.alloc.alloc()
        self.pool.state[s].copy_(prefill_state.to(self.device, torch.float32))
        dl.dl_reset_slots(self.pool, torch.tensor([s], dtype=torch.int32, device=self.device))
        rid = self._next_rid
        self._next_rid += 1
        self.requests[rid] = Request(rid, s)
        self.active.append(rid)
        self._membership_changed()
        return rid

    def retire(self, rid: int) -> Request:
        """The request leaves the batch; its slot returns to the free list."""
        r = self.requests.pop(rid)
        self.active.remove(rid)
        self.alloc.free(r.slot)
        self._membership_changed()
        return r

    def set_lambda_per_head(self, layer: int, lam: torch.Tensor):
        """Per-head constant log-decays of a layer ([H] or [H, d_k]; RetNet)."""
        if not self.lambda_per_head:
            raise ValueError("the server was made without per-head constant decays")
        self.lam_const[layer] = lam.to(self.device, torch.float32).contiguous()
        self._graphs.clear()
        self._prepared.clear()

    def _membership_changed(self):
        B = len(self.active)
        if B:
            ids = torch.tensor([self.requests[r].slot for r in self.active], dtype=torch.int32)
            self.slots_buf[:B].copy_(ids, non_blocking=True)

    # -- decode --------------------------------------------------------------------
    def _calls(self, B: int):
        if B not in self._prepared:
            steps = []
            for l, b in enumerate(self.bufs):
                lam = self.lam_const[l] if self.lambda_per_head else (None if b["lam"] is None else b["lam"][:B])
                steps.append(dl.PreparedStep("decode", self.pool, l, self.slots_buf[:B], b["q"][:B], b["k"][:B],
                                             b["v"][:B], lam, None if b["beta"] is None else b["beta"][:B],
                                             b["out"][:B], self.lambda_per_head, auto_merge=self.merge))
            self._prepared[B] = steps
        return self._prepared[B]

    def _launch(self, B: int):
        for p in self._calls(B):
            st = p()
            if st != dl.DL_OK:
                raise dl.DeltaLogError(st, "dl_decode_step")

    def _check_inputs(self, inputs, B: int):
        """Every input the server's operator needs, for every layer, with exactly the
        rows of the active requests (no broadcasting into the step buffers)."""
        if len(inputs) != self.n_layers:
            raise ValueError(f"expected inputs for {self.n_layers} layers, got {len(inputs)}")
        for l, x in enumerate(inputs):
            b = self.bufs[l]
            for key in ("q", "k", "v", "lam", "beta"):
                if b[key] is None:
                    if x.get(key) is not None:
                        raise ValueError(f"layer {l}: this server takes no '{key}' per step")
                    continue
                if x.get(key) is None:
                    raise ValueError(f"layer {l}: '{key}' is missing")
                want = tuple(b[key][:B].shape)
                if tuple(x[key].shape) != want:
                    raise ValueError(f"layer {l}: '{key}' must be {list(want)}, got {list(x[key].shape)}")

    def step(self, inputs) -> list[torch.Tensor]:
        """One decode step of every active request over all layers.  ``inputs[l]`` holds
        layer l's rows.  Returns each layer's outputs [B, H, d_v] (views of the server's
        buffers, valid until the next step)."""
        B = len(self.active)
        if B == 0:
            return []
        self._check_inputs(inputs, B)
        for l, x in enumerate(inputs):
            b = self.bufs[l]
            for key in ("q", "k", "v", "lam", "beta"):
                if b[key] is not None:
                    b[key][:B].copy_(x[key], non_blocking=True)
        if self.use_graphs:
            g = self._graphs.get(B)
            if g is None:
                self._launch(B)   # first use of this batch size runs directly (and sets kernels up)
                g = torch.cuda.CUDAGraph()
                cs = torch.cuda.Stream()
                cs.wait_stream(torch.cuda.current_stream())
                with torch.cuda.stream(cs):
                    g.capture_begin(capture_error_mode="thread_local")
                    self._launch(B)
                    g.capture_end()
                torch.cuda.current_stream().wait_stream(cs)
                self._graphs[B] = g
            else:
                g.replay()
        else:
            self._launch(B)
        for rid in self.active:
            self.requests[rid].steps += 1
        return [b["out"][:B] for b in self.bufs]

    def errors(self) -> int:
        return dl.dl_read_error(self.pool)
