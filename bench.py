#!/usr/bin/env python
"""Benchmark of the base + log recurrent-state decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--log-cap L] [--batch B] [--subs LIST] [--merge-legs LIST]

A step is one decode step of the whole batch over all layers of the workload (one
library call per layer), with every slot advancing by one token; merges happen on
each slot's own merge step inside the same call.  Inputs are seeded synthetic
tensors resident in HBM before timing starts.

The headline workload is the largest one: KDA-style per-key decay with the delta
rule, 24 layers x batch 256 x 32 heads, d = 128, log capacity L = 16 (12 GiB of
base state).  Slot phases are spread (``--phases spread``, default): slot b of slot
group g starts its merge cycle at offset (o_b + g * batch) mod L, o_b = b (or the
workload's own random stagger, RetNet), so every launch of a batch of at least L
slots carries exactly its 1/L share of merge steps and any window of timed steps is
the amortised step.  The JSON line records the live-entry histogram of the timed
launches.  ``--phases workload`` keeps the workload's own offsets for every group.

Besides the headline, the line carries sub-records (``--subs``), each with its own
steps/s, roofline and eager comparison, and merge legs (``--merge-legs``) that time
standalone ``dl_merge`` of full logs and ``dl_materialize``.  A sub-record's step
count is at least K, raised so its timed region is a few ms, and a multiple of L.

Cold L2 between steps, two ways (``--l2``):
  rotate (default)  inputs larger than L2: the pool holds R disjoint copies of the
                    batch's slots, stepped in turn (step j uses group j mod R), with R
                    the smallest count whose base states total >= 384 MiB (three times
                    the 126 MB L2); R = 1 when one step's state is that large already.
                    A step's state was last touched >= 2 L2-sizes of traffic earlier.
                    The K steps run back to back between one pair of CUDA events,
                    launched from a CUDA graph (``--launch graph``, default) or
                    directly (``--launch stream``).
  flush             before every timed step, outside the timed interval, L2 is
                    flushed by writing a 256 MiB buffer and then reading a second
                    256 MiB buffer (the read evicts the dirty lines the write left);
                    each step is bracketed by its own CUDA events.

Multi-GPU (torchrun, one process per GPU): the slots are independent, so each rank
runs its own replica of the workload (weak scaling, no collective on the data
path); the reported time is the max over ranks.

Prints one JSON line (rank 0).  ``--impl reference`` times the fp64 CPU oracle of
the eager recurrence on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "decode head-steps/s (batch x heads x layers)"
UNIT = "head-steps/s"
FLUSH_BYTES = 256 << 20
ROTATE_MIN_BYTES = 384 << 20  # base-state bytes of one rotation: three times L2 (126 MB)
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "dram_traffic.txt")
CSRC = os.path.join(ROOT, "recurrent_state_serving_b200", "csrc")
DEFAULT_WORKLOAD = "kda_diag_delta"
DEFAULT_SUBS = ("gla_rwkv6_diag:b64:L8,retnet_scalar:b64,retnet_scalar:b256,retnet_scalar:b1024,gdn_gva:b1,"
                "retnet_scalar:b1,retnet_scalar:b16")
DEFAULT_MERGE_LEGS = "kda_diag_delta,retnet_scalar:b256"
SUB_MIN_MS = 3.0            # a sub-record's timed region is at least about this long
SUB_MAX_STEPS = 4096
HOST_INPUT_BYTES = 128 << 20  # distinct seeded steps generated per workload (host side)
DELTA_READING = ("decayed state: b_t = beta_t (v_t - (Diag(exp lambda_t) S_{t-1})^T k_t), "
                 "the gated delta rule of GDN/KDA (DL_UPDATE_DELTA)")


def kernel_source_hash() -> str:
    """Hash of the CUDA sources; a recorded ncu traffic figure is only valid for it."""
    h = hashlib.sha256()
    for f in sorted(os.listdir(CSRC)):
        h.update(f.encode())
        h.update(open(os.path.join(CSRC, f), "rb").read())
    return h.hexdigest()[:16]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=32)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--log-cap", type=int, default=None)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--layers", type=int, default=None,
                    help="override the workload's layer count (small cases for profiling)")
    ap.add_argument("--subs", default=DEFAULT_SUBS,
                    help="comma list of name[:bB][:LL] sub-records, or 'none'")
    ap.add_argument("--merge-legs", default=DEFAULT_MERGE_LEGS,
                    help="comma list of name[:bB][:LL] workloads whose dl_merge/dl_materialize are timed, or 'none'")
    ap.add_argument("--phases", default="spread", choices=["spread", "workload"],
                    help="slot merge phases: spread over each launch, or the workload's own offsets")
    ap.add_argument("--merge", default="adaptive", choices=["adaptive", "capacity"],
                    help="dl_decode_step merge policy: adaptive (launches too small to fill the GPU "
                         "merge every step) or capacity (every slot merges on its L-th step)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-eager", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--traffic-from", default=None,
                    help="append a record to profiles/dram_traffic.txt from an ncu csv and exit")
    ap.add_argument("--traffic-kind", default="decode", choices=["decode", "eager", "merge", "materialize"],
                    help="which launches an ncu csv given with --traffic-from holds")
    ap.add_argument("--tile-v", type=int, default=0,
                    help="work-unit width: 0 automatic, 16/32 value tiles, 128 whole heads")
    ap.add_argument("--l2", default="rotate", choices=["rotate", "flush"],
                    help="cold L2 per step: rotate slot groups (inputs > L2) or flush before each step")
    ap.add_argument("--launch", default="graph", choices=["graph", "stream"],
                    help="rotate mode: replay the timed steps from a CUDA graph or launch them directly")
    ap.add_argument("--replay", default="per_tile", choices=["per_tile", "cluster"],
                    help="value-tiled kernel: ReplayPrep formed per tile, or shared by a head's tiles as one cluster")
    ap.add_argument("--e2e-copies", default="packed", choices=["packed", "per_tensor"],
                    help="end-to-end leg: copy each input/output tensor, or one packed buffer per step")
    ap.add_argument("--log-format", default="fp32", choices=["fp32", "compact"],
                    help="log entry layout: fp32 [a|b|Lambda], or compact (bf16 a, bf16 b without the delta rule)")
    return ap.parse_args(argv)


def parse_spec(spec: str):
    """'name[:bB][:LL][:nN]' -> a synth workload with that batch / log capacity / layer count."""
    from recurrent_state_serving_b200 import synth
    parts = spec.strip().split(":")
    if parts[0] not in synth.WORKLOADS:
        raise SystemExit(f"unknown workload {parts[0]!r} (known: {', '.join(sorted(synth.WORKLOADS))})")
    wl = synth.WORKLOADS[parts[0]]
    for p in parts[1:]:
        if p.startswith("b"):
            wl = wl.with_(batch=int(p[1:]))
        elif p.startswith("L"):
            wl = wl.with_(log_cap=int(p[1:]))
        elif p.startswith("n"):
            wl = wl.with_(n_layers=int(p[1:]))
        else:
            raise SystemExit(f"bad workload spec {spec!r}")
    return wl


def spec_list(text: str):
    if not text or text.strip().lower() == "none":
        return []
    return [parse_spec(s) for s in text.split(",") if s.strip()]


def workload(a):
    wl = parse_spec(a.workload)
    if a.log_cap:
        wl = wl.with_(log_cap=a.log_cap)
    if a.batch:
        wl = wl.with_(batch=a.batch)
    if a.layers:
        wl = wl.with_(n_layers=a.layers)
    return wl


def rotation_groups(wl, l2_mode: str) -> int:
    """Slot groups stepped in turn so that the base states of one rotation total at
    least ROTATE_MIN_BYTES (1 under the flush method, or when one step's are enough)."""
    if l2_mode == "flush":
        return 1
    step_state = wl.units_per_step * 4 * wl.d_k * wl.d_v
    return max(1, -(-ROTATE_MIN_BYTES // step_state))


def phase_offsets(wl, n_groups: int, mode: str = "spread") -> np.ndarray:
    """Staggering offsets [n_groups, batch]: how many untimed steps each slot of each
    group takes before the common steps.

    spread    slot b of group g: (o_b + g * batch) mod L with o_b = b, or the
              workload's own random offset when it is staggered.  A batch of at least
              L slots (and o_b = b) then holds every live length 0..L-1 equally in
              every launch; smaller batches continue the phase sequence across groups.
    workload  the workload's own offsets (zeros unless staggered) for every group."""
    from recurrent_state_serving_b200 import synth
    own = synth.slot_offsets(wl)
    if mode == "workload":
        return np.tile(own, (n_groups, 1))
    if mode != "spread":
        raise ValueError(mode)
    base = own if wl.staggered else np.arange(wl.batch)
    g = np.arange(n_groups)[:, None]
    return ((base[None, :] + g * wl.batch) % wl.log_cap).astype(np.int64)


def live_entries(offsets, step_index: int, n_groups: int, log_cap: int):
    """Live log entries each slot of the group stepped at global step ``step_index``
    holds when the step starts: that group has taken step_index // n_groups steps
    before it, after its staggering pre-steps (the same offsets for every group)."""
    return (offsets + step_index // n_groups) % log_cap


def group_live_entries(group_offsets, step_index: int, log_cap: int):
    """live_entries() with each group's own offsets ([n_groups, batch])."""
    R = group_offsets.shape[0]
    return (group_offsets[step_index % R] + step_index // R) % log_cap


def expected_live_lengths(wl, group_offsets, n_steps: int, merge_every: bool = False):
    """Live entries of every slot of every group ([n_groups, batch]) after global steps
    0 .. n_steps-1 (step j on group j mod R), as the byte accounting assumes.  Merging
    every step, a group keeps its pre-step live lengths until its first step."""
    R = group_offsets.shape[0]
    taken = np.array([(n_steps - g + R - 1) // R for g in range(R)])
    if merge_every:
        return np.where(taken[:, None] > 0, 0, group_offsets)
    return (group_offsets + taken[:, None]) % wl.log_cap


def timed_window_bytes(wl, group_offsets, first: int, K: int, log_format: str = "fp32",
                       merge_every: bool = False):
    """Algorithmic bytes of global steps first .. first+K-1 (all layers and heads)
    and the histogram of the slots' live entries at those steps.  merge_every: the
    launches merge every slot on every step (the adaptive policy on a small launch),
    so every slot enters with an empty log and takes the merge step."""
    from recurrent_state_serving_b200 import traffic
    L = wl.log_cap
    scale = wl.n_heads * wl.n_layers
    hist = np.zeros(L, np.int64)
    if merge_every:
        # a group's first step folds its pre-step entries; every later step starts empty
        R = group_offsets.shape[0]
        for j in range(first, first + K):
            c = group_offsets[j % R] if j // R == 0 else np.zeros(wl.batch, np.int64)
            hist += np.bincount(c, minlength=L)
        per_c = [traffic.deferred_head_step(wl, c, merge=True, log_format=log_format) for c in range(L)]
        return float(np.dot(hist, per_c)) * scale, hist
    per_c = [traffic.deferred_head_step(wl, c, merge=(c == L - 1), log_format=log_format) for c in range(L)]
    for j in range(first, first + K):
        hist += np.bincount(group_live_entries(group_offsets, j, L), minlength=L)
    per_slot = float(np.dot(hist, per_c))
    return per_slot * scale, hist


def sub_steps(wl, K: int, log_format: str = "fp32") -> int:
    """Timed steps of a sub-record: at least K, enough for about SUB_MIN_MS at 5 TB/s
    (plus 3 us per launch), a multiple of L, at most SUB_MAX_STEPS."""
    from recurrent_state_serving_b200 import traffic
    est_ms = (traffic.deferred_cycle_average(wl, log_format) * wl.units_per_step / 5e12 * 1e3
              + 3e-3 * wl.n_layers)
    n = max(K, int(math.ceil(SUB_MIN_MS / est_ms)))
    n = -(-n // wl.log_cap) * wl.log_cap
    return min(n, max(K, SUB_MAX_STEPS))


def distinct_steps(wl) -> int:
    """Distinct seeded input steps generated for a workload (cycled while timing)."""
    from recurrent_state_serving_b200 import traffic
    per = traffic.token_bytes(wl) * wl.units_per_step
    return int(max(2, min(wl.steps, 256 // wl.n_layers, HOST_INPUT_BYTES // max(1.0, per))))


def l2_description(wl, l2_mode: str, launch: str) -> str:
    if l2_mode == "flush":
        return ("flushed before every timed step, outside the timed interval: 256 MiB write, then "
                "256 MiB read of another buffer (evicts the dirty lines); per-step CUDA events")
    R = rotation_groups(wl, l2_mode)
    mib = R * wl.units_per_step * 4 * wl.d_k * wl.d_v / 2**20
    return (f"inputs larger than L2: {R} slot group(s) of the batch stepped in turn, {mib:.0f} MiB of "
            f"base state per rotation (L2 126 MB); timed steps back to back, "
            f"{'replayed from one CUDA graph' if launch == 'graph' else 'launched directly'}")


def phases_description(wl, mode: str) -> str:
    if mode == "workload":
        return ("each group keeps the workload's own offsets: "
                + ("random in [0, L) per slot" if wl.staggered else "all slots merge on the same step"))
    src = "the workload's random offset o_b in [0, L)" if wl.staggered else "o_b = b"
    return (f"spread: slot b of group g starts its merge cycle at (o_b + g*batch) mod L, {src}; "
            f"every launch of >= L slots holds each live length 0..L-1 equally")


def config_of(wl, n_gpus, tile_v=0, l2_mode="rotate", launch="graph", log_format="fp32", replay="per_tile",
              phases="spread"):
    suffix = "" if log_format == "fp32" else f"_{log_format}log"
    cfg = {"workload": f"{wl.name}_b{wl.batch}_h{wl.n_heads}_d{wl.d_k}_L{wl.log_cap}{suffix}",
           "tile_v": tile_v or "auto", "log_format": log_format, "replay": replay,
           "layers": wl.n_layers, "batch_per_gpu": wl.batch, "heads": wl.n_heads,
           "kheads": wl.n_kheads, "d_k": wl.d_k, "d_v": wl.d_v, "log_cap": wl.log_cap,
           "decay": wl.decay, "update": wl.update, "inputs": wl.in_dtype, "state": "fp32",
           "phases": phases_description(wl, phases),
           "l2": l2_description(wl, l2_mode, launch),
           "parallelism": f"replicas x{n_gpus} (independent slots, no collective)"}
    if wl.update == "delta":
        cfg["delta_reading"] = DELTA_READING
    return cfg


def workload_key(wl, log_format="fp32") -> str:
    return config_of(wl, 1, log_format=log_format)["workload"]


def traffic_summary_from_ncu(csv_path: str, workload_key: str, kernel_regex: str, kind: str = "decode") -> str:
    """One record for profiles/dram_traffic.txt from an ncu --csv export of
    dram__bytes_read.sum and dram__bytes_write.sum (and, when present, the L2 write
    sectors lts__t_sectors_srcunit_tex_op_write.sum) over consecutive launches of
    one kernel.  For decode launches the capture should span a whole cycle of
    launch mixes, so append and merge heads mix as in the timed region.
    Run: python bench.py --traffic-from <csv> --traffic-kind KIND [--workload ...]."""
    import csv
    import re
    rows = list(csv.reader(open(csv_path)))
    i = [k for k, r in enumerate(rows) if "Kernel Name" in r][0]
    hdr = rows[i]
    kn, mn, mv = hdr.index("Kernel Name"), hdr.index("Metric Name"), hdr.index("Metric Value")
    mu = hdr.index("Metric Unit") if "Metric Unit" in hdr else None
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9,
             "sector": 1, "Ksector": 1e3, "Msector": 1e6, "Gsector": 1e9}
    per, l2w = {}, {}
    idcol = hdr.index("ID") if "ID" in hdr else None
    for r in rows[i + 1:]:
        if len(r) <= mv or not re.search(kernel_regex, r[kn]):
            continue
        key = r[idcol] if idcol is not None else len(per)
        v = float(r[mv].replace(",", "")) * scale.get(r[mu] if mu is not None else "byte", 1)
        if r[mn] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            per[key] = per.get(key, 0.0) + v
        elif r[mn] == "lts__t_sectors_srcunit_tex_op_write.sum":
            l2w[key] = l2w.get(key, 0.0) + 32.0 * v
    vals = list(per.values())
    if not vals:
        raise SystemExit("no matching launches in " + csv_path)
    avg = sum(vals) / len(vals)
    text = (f"workload = {workload_key}\nkind = {kind}\nkernel_sha = {kernel_source_hash()}\n"
            f"launches = {len(vals)}\ndram_bytes_per_launch = {avg:.0f}\n"
            f"min_launch_bytes = {min(vals):.0f}\nmax_launch_bytes = {max(vals):.0f}\n")
    if l2w:
        text += f"l2_write_bytes_per_launch = {sum(l2w.values()) / len(l2w):.0f}\n"
    return text


def traffic_records(path=None):
    """Records of profiles/dram_traffic.txt: each starts at a 'workload = ' line."""
    path = path or PROFILE_TRAFFIC
    if not os.path.exists(path):
        return []
    recs, cur = [], None
    for line in open(path):
        if "=" not in line or line.lstrip().startswith("#"):
            continue
        k, v = (x.strip() for x in line.split("=", 1))
        if k == "workload":
            cur = {}
            recs.append(cur)
        if cur is not None:
            cur[k] = v
    return recs


def recorded_traffic(workload_key, kind="decode", field="dram_bytes_per_launch"):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, or None
    when there is none for this workload and kind, or the kernel source changed
    since it was taken."""
    sha = kernel_source_hash()
    for r in traffic_records():
        if r.get("workload") != workload_key or r.get("kind", "decode") != kind:
            continue
        if r.get("kernel_sha") != sha:
            continue
        try:
            return float(r[field])
        except (KeyError, ValueError):
            return None
    return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy)"
    return 6650.0, "fallback (6.65 TB/s)"


# ---------------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.rows = []
        self.windows = []
        self.proc = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            self.sel = ["-i", str(device_index)]

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *self.sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        inside = [r for (t, r) in self.rows if any(a - 0.05 <= t <= b + 0.05 for a, b in self.windows)]
        rows = inside or [r for _, r in self.rows]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[0]))
                smax.append(float(r[1]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, r[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm), "samples_in_timed_windows": len(inside)}


# ---------------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------------
def res_kernel_name(wl, tile_v):
    whole = tile_v == 128 or (tile_v == 0 and wl.d_k == 128 and wl.d_v == 128
                              and wl.batch * wl.n_heads >= 148)
    return "dl::wh::warp_head_kernel" if whole else "dl::step_kernel"


def max_over_ranks(x: float, dist=None, device=None) -> float:
    """Max of a per-rank scalar over all ranks (the timing rule for multi-GPU runs)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


def graph_upload(graph, stream) -> bool:
    """Upload an instantiated CUDA graph to the device ahead of its first replay, so
    the replay inside the timed interval carries no upload work."""
    import ctypes
    try:
        rt = ctypes.CDLL("libcudart.so.12")
        ex = graph.raw_cuda_graph_exec()
        if not isinstance(ex, int):
            get = ctypes.pythonapi.PyCapsule_GetPointer
            get.restype, get.argtypes = ctypes.c_void_p, [ctypes.py_object, ctypes.c_char_p]
            ex = get(ex, None)
        rt.cudaGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        return rt.cudaGraphUpload(ctypes.c_void_p(ex), ctypes.c_void_p(stream.cuda_stream)) == 0
    except (OSError, AttributeError, TypeError, ValueError):
        return False


# ---------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------
PACK_ALIGN = 256


def pack_layout(spec, align: int = PACK_ALIGN):
    """Byte offsets of a step's tensors packed into one buffer.

    spec: one dict per layer, {name: (shape, dtype) or None}.  Each tensor starts on
    an ``align``-byte boundary.  Returns (total bytes, one {name: offset or None}
    dict per layer)."""
    off, offs = 0, []
    for layer in spec:
        d = {}
        for k, v in layer.items():
            if v is None:
                d[k] = None
                continue
            shape, dtype = v
            n = int(np.prod(shape)) * torch_elem_size(dtype)
            off = -(-off // align) * align
            d[k] = off
            off += n
        offs.append(d)
    return -(-off // align) * align, offs


def torch_elem_size(dtype) -> int:
    import torch
    return torch.empty((), dtype=dtype).element_size()


def packed_views(buf, spec, offs):
    """Typed views of a uint8 buffer laid out by pack_layout."""
    out = []
    for layer, o in zip(spec, offs):
        d = {}
        for k, v in layer.items():
            if v is None:
                d[k] = None
                continue
            shape, dtype = v
            n = int(np.prod(shape)) * torch_elem_size(dtype)
            d[k] = buf[o[k]:o[k] + n].view(dtype).view(shape)
        out.append(d)
    return out


class GpuContext:
    """Device, ranks, clocks and the timing loop shared by every leg."""

    def __init__(self, a, world, dist):
        import torch
        self.torch = torch
        self.a, self.world, self.dist = a, world, dist
        self.dev = torch.device("cuda", torch.cuda.current_device())
        self.sampler = ClockSampler(self.dev.index)
        self.sampler.start()
        self.launches = 0
        if a.l2 == "flush":
            self.flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=self.dev)
            self.flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=self.dev)
            self.flush_sink = torch.empty((), dtype=torch.float32, device=self.dev)
        self.graph_uploaded = None

    def flush_l2(self):
        self.flush.zero_()
        self.torch.sum(self.flush_rd, dim=0, out=self.flush_sink)

    def barrier_sync(self):
        self.torch.cuda.synchronize()
        if self.dist is not None:
            self.dist.barrier()
        self.torch.cuda.synchronize()

    def reduce_max(self, x):
        return max_over_ranks(x, self.dist, self.dev)

    def timed(self, calls_for_step, n_steps, W, graph_ok=True, per_step_events=False):
        """calls_for_step(j) -> callables issued for global step j.  Steps 0..W-1 run
        untimed, W..W+n_steps-1 timed.  Returns the timed interval in ms (the sum of
        per-step intervals when flushing or with per_step_events)."""
        torch = self.torch
        a = self.a
        for j in range(W):
            for c in calls_for_step(j):
                c()
        self.barrier_sync()
        if a.l2 == "flush" or per_step_events:
            t0 = time.time()
            evs = []
            for i in range(n_steps):
                if a.l2 == "flush":
                    self.flush_l2()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                for c in calls_for_step(W + i):
                    c()
                e1.record()
                evs.append((e0, e1))
            self.barrier_sync()
            self.sampler.mark(t0, time.time())
            return sum(e0.elapsed_time(e1) for e0, e1 in evs)
        g = None
        if a.launch == "graph" and graph_ok:
            g = torch.cuda.CUDAGraph()
            cs = torch.cuda.Stream()
            cs.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(cs):
                g.capture_begin(capture_error_mode="thread_local")
                for i in range(n_steps):
                    for c in calls_for_step(W + i):
                        c()
                g.capture_end()
            torch.cuda.current_stream().wait_stream(cs)
            up = graph_upload(g, torch.cuda.current_stream())
            self.graph_uploaded = up if self.graph_uploaded is None else (self.graph_uploaded and up)
            self.barrier_sync()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        t0 = time.time()
        e0.record()
        if g is not None:
            g.replay()
        else:
            for i in range(n_steps):
                for c in calls_for_step(W + i):
                    c()
        e1.record()
        self.barrier_sync()
        self.sampler.mark(t0, time.time())
        ms = e0.elapsed_time(e1)
        del g
        return ms


def check_status(st, what="dl_decode_step"):
    if st != 0:
        from recurrent_state_serving_b200 import deltalog as dl
        raise dl.DeltaLogError(st, what)


class WorkloadSetup:
    """A workload's distinct seeded inputs on the device and its output buffers."""

    def __init__(self, ctx, wl):
        from recurrent_state_serving_b200 import synth
        from recurrent_state_serving_b200.runner import _to_dev_input
        torch = ctx.torch
        self.wl = wl
        self.ndist = distinct_steps(wl)
        self.host = [[synth.step_inputs(wl, t, l) for l in range(wl.n_layers)] for t in range(self.ndist)]
        self.dev = [[{k: _to_dev_input(v, wl.in_dtype if k in ("q", "k", "v") else "f32", ctx.dev)
                      for k, v in x.items()} for x in per_layer] for per_layer in self.host]
        self.outs = [torch.empty(wl.batch, wl.n_heads, wl.d_v, dtype=torch.float32, device=ctx.dev)
                     for _ in range(wl.n_layers)]

    def prestep_inputs(self, p, layer):
        return self.dev[p % self.ndist][layer]


def prepared_calls(kind, wl, runner, setup, R, cache, merge="capacity"):
    """Step j: group j mod R, distinct inputs j mod ndist (argument blocks built once)."""
    from recurrent_state_serving_b200 import deltalog as dl

    def calls(j):
        key = (j % R, j % setup.ndist)
        if key not in cache:
            g, t = key
            cache[key] = [dl.PreparedStep(kind, runner.pool, l, runner.group_slots[g], x["q"], x["k"],
                                          x["v"], x["lam"], x["beta"], setup.outs[l], wl.lambda_const,
                                          auto_merge=merge)
                          for l, x in enumerate(setup.dev[t])]
        return [(lambda p=p: check_status(p())) for p in cache[key]]
    return calls


def roofline_record(achieved_gbs, kernel, launches, total_ms, bytes_per_launch, traffic_bytes):
    peak, peak_src = measured_peaks()
    return {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved_gbs / peak, 4), "peak_source": peak_src,
            "traffic": traffic_bytes, "algorithmic_bytes_per_launch": round(bytes_per_launch),
            "kernel": kernel, "launches_timed": launches,
            "avg_launch_us": round(total_ms * 1e3 / launches, 3),
            "frac_of_8tbs_spec": round(achieved_gbs / 8000.0, 4)}


def decode_leg(ctx, wl, K, W, setup, merge):
    """Timed deferred decode steps under one merge policy.  Returns (record, runner,
    rotation groups, group offsets)."""
    from recurrent_state_serving_b200 import deltalog as dl
    from recurrent_state_serving_b200 import traffic
    from recurrent_state_serving_b200.runner import DecodeRunner
    a = ctx.a
    R = rotation_groups(wl, a.l2)
    goffs = phase_offsets(wl, R, a.phases)
    r = DecodeRunner(wl, device=str(ctx.dev), tile_v=a.tile_v, n_groups=R, log_format=a.log_format,
                     replay=a.replay, offsets=goffs, merge=merge)
    every = dl.dl_merge_policy(wl.batch, wl.n_heads, merge)
    r.load_initial_state(on_device=True)
    r.run_presteps(inputs=setup.prestep_inputs)
    total_ms = ctx.timed(prepared_calls("decode", wl, r, setup, R, {}, merge), K, W)
    if r.errors() != 0:
        raise RuntimeError("device error bits set during the benchmark")
    # the slots' live lengths must be the ones the byte accounting assumes
    live = np.stack([r.pool.log_len[gs.long(), 0].cpu().numpy() for gs in r.group_slots])
    want = expected_live_lengths(wl, goffs, W + K, every)
    if not np.array_equal(live, want):
        raise RuntimeError(f"slot phases differ from the byte model in {int((live != want).sum())} slots")
    max_ms = ctx.reduce_max(total_ms)
    launches = K * wl.n_layers
    ctx.launches += launches
    bytes_total, hist = timed_window_bytes(wl, goffs, W, K, a.log_format, merge_every=every)
    achieved = bytes_total / (total_ms / 1e3) / 1e9
    key = workload_key(wl, a.log_format)
    units = hist.sum() * wl.n_heads * wl.n_layers
    kernel = "dl::step_kernel (merging every step)" if every else res_kernel_name(wl, a.tile_v)
    rec = {"workload": key, "merge_policy": merge, "merges_every_step": every,
           "value": whole_job_rate(wl.units_per_step * K, ctx.world, max_ms), "unit": UNIT,
           "ms_per_step": max_ms / K, "steps": K, "warmup": W, "rotation_groups": R,
           "roofline": roofline_record(achieved, kernel, launches, total_ms,
                                       bytes_total / launches,
                                       None if every else recorded_traffic(key, "decode")),
           "live_entries": {"hist": [int(x) for x in hist],
                            "merge_share": 1.0 if every else round(float(hist[-1]) / max(1, hist.sum()), 4),
                            "bytes_per_head_step": round(bytes_total / units, 1),
                            "cycle_average_model": round(traffic.deferred_cycle_average(wl, a.log_format), 1)},
           "deferred_bytes_per_step": round(bytes_total / K)}
    return rec, r, R, goffs


def measure_decode(ctx, wl, K, W, *, eager=True, keep=False):
    """Deferred decode steps of a workload (the product path, merge policy --merge),
    then the in-library eager step on the same workload; when the adaptive policy
    merges every step (a small launch), also the at-capacity policy.  Returns
    (record, runner and setup when keep)."""
    from recurrent_state_serving_b200 import traffic
    from recurrent_state_serving_b200.runner import DecodeRunner
    torch = ctx.torch
    a = ctx.a
    setup = WorkloadSetup(ctx, wl)
    rec, r, R, goffs = decode_leg(ctx, wl, K, W, setup, a.merge)
    key = rec["workload"]
    bytes_total = rec["deferred_bytes_per_step"] * K
    launches = K * wl.n_layers
    if rec["merges_every_step"]:
        cap, r_cap, _, _ = decode_leg(ctx, wl, K, W, setup, "capacity")
        rec["at_capacity"] = {k: cap[k] for k in ("value", "ms_per_step", "roofline", "live_entries")}
        del r_cap
    if wl.update == "delta":
        rec["delta_reading"] = DELTA_READING
    if eager and not a.no_eager:
        re_ = DecodeRunner(wl, device=str(ctx.dev), mode="eager", tile_v=a.tile_v, n_groups=R)
        re_.load_initial_state(on_device=True)
        ms_e = ctx.timed(prepared_calls("eager", wl, re_, setup, R, {}), K, W)
        if re_.errors() != 0:
            raise RuntimeError("device error bits set in the eager leg")
        ctx.launches += launches
        tot_e = ctx.reduce_max(ms_e)
        eb = traffic.eager_head_step(wl) * wl.units_per_step * K
        ach_e = eb / (ms_e / 1e3) / 1e9
        rec["eager"] = {"value": whole_job_rate(wl.units_per_step * K, ctx.world, tot_e),
                        "ms_per_step": tot_e / K, "algorithmic_bytes_per_step": round(eb / K),
                        "achieved_gbs": round(ach_e, 1), "frac": round(ach_e / measured_peaks()[0], 4),
                        "kernel": "dl::step_kernel (eager flag)",
                        "traffic": recorded_traffic(key, "eager")}
        rec["deferred_over_eager"] = round(rec["value"] / rec["eager"]["value"], 3)
        rec["eager_bytes_over_deferred"] = round(eb / bytes_total, 3)
        del re_
    if keep:
        return rec, (r, setup, R, goffs)
    del r, setup
    torch.cuda.empty_cache()
    return rec, None


def measure_merge(ctx, wl, K, W):
    """Standalone merge (dl_merge of full logs, c = L on every head) and materialise
    (dl_materialize of the same logs, pool unchanged), all layers per step."""
    from recurrent_state_serving_b200 import deltalog as dl
    from recurrent_state_serving_b200 import traffic
    from recurrent_state_serving_b200.runner import DecodeRunner
    torch = ctx.torch
    a = ctx.a
    setup = WorkloadSetup(ctx, wl)
    R = rotation_groups(wl, a.l2)
    r = DecodeRunner(wl, device=str(ctx.dev), tile_v=a.tile_v, n_groups=R, log_format=a.log_format,
                     replay=a.replay, offsets=np.zeros((R, wl.batch), np.int64))
    r.load_initial_state(on_device=True)
    L = wl.log_cap
    appends = {}

    def fill(g):
        # L appends per layer: every head of the group holds a full log (c = L)
        for t in range(L):
            key = (g, t % setup.ndist)
            if key not in appends:
                x_l = setup.dev[t % setup.ndist]
                appends[key] = [dl.PreparedStep("append", r.pool, l, r.group_slots[g], x["q"], x["k"], x["v"],
                                                x["lam"], x["beta"], None, wl.lambda_const)
                                for l, x in enumerate(x_l)]
            for p in appends[key]:
                check_status(p(), "dl_append")

    dense = torch.empty(wl.batch, wl.n_heads, wl.d_k, wl.d_v, dtype=torch.float32, device=ctx.dev)
    # materialise first (the pool is not changed): back-to-back steps over full logs
    for g in range(R):
        fill(g)

    def mat_calls(j):
        g = j % R
        return [(lambda l=l: dl.dl_materialize(r.pool, l, r.group_slots[g], dense)) for l in range(wl.n_layers)]
    ms_m = ctx.timed(mat_calls, K, W, graph_ok=False)
    # merge: each timed step folds one group's full logs; refills are untimed
    ms_g = 0.0
    for i in range(W + K):
        g = i % R
        if i >= R:
            fill(g)
        torch.cuda.synchronize()
        if a.l2 == "flush":
            ctx.flush_l2()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        t0 = time.time()
        e0.record()
        for l in range(wl.n_layers):
            dl.dl_merge(r.pool, l, r.group_slots[g])
        e1.record()
        torch.cuda.synchronize()
        if i >= W:
            ctx.sampler.mark(t0, time.time())
            ms_g += e0.elapsed_time(e1)
    if r.errors() != 0:
        raise RuntimeError("device error bits set in the merge leg")
    if int(r.pool.log_len.abs().sum()) != 0 and R == 1:
        raise RuntimeError("merge left live entries")
    launches = K * wl.n_layers
    ctx.launches += 2 * launches
    per_head = traffic.merge_head(wl, L, a.log_format)
    tot = per_head * wl.units_per_step * K
    key = workload_key(wl, a.log_format)
    out = {}
    for name, ms in (("merge", ctx.reduce_max(ms_g)), ("materialize", ctx.reduce_max(ms_m))):
        ach = tot / (ms / 1e3) / 1e9
        out[name] = {"value": whole_job_rate(wl.units_per_step * K, ctx.world, ms), "unit": "head-merges/s",
                     "ms_per_step": ms / K, "live_entries": L,
                     "roofline": roofline_record(ach, "dl::merge_kernel", launches, ms, tot / launches,
                                                 recorded_traffic(key, name))}
    del r, setup, dense
    torch.cuda.empty_cache()
    return {"workload": key, "bytes_per_head": per_head,
            "calls": "dl_merge / dl_materialize per layer, every head with c = L live entries", **out}


def measure_e2e(ctx, wl, K, W, runner, setup, R, goffs):
    """End to end through the public API with host buffers: pinned host inputs ->
    H2D -> dl_decode_step per layer -> D2H of o_t, all inside the events."""
    from recurrent_state_serving_b200 import deltalog as dl
    torch = ctx.torch
    a = ctx.a
    dev = ctx.dev
    r = runner
    outs = setup.outs
    if a.e2e_copies == "packed":
        spec = [{k: (None if v is None else (tuple(v.shape), v.dtype)) for k, v in x.items()}
                for x in setup.dev[0]]
        in_bytes, in_offs = pack_layout(spec)
        host_pk = []
        for per_layer in setup.dev:
            hb = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
            for view, x in zip(packed_views(hb, spec, in_offs), per_layer):
                for k, v in x.items():
                    if v is not None:
                        view[k].copy_(v.cpu())
            host_pk.append(hb)
        out_spec = [{"o": (tuple(o.shape), o.dtype)} for o in outs]
        out_bytes, out_offs = pack_layout(out_spec)
        h2d, d2h = in_bytes, out_bytes   # the buffers copied (tensors plus alignment padding)
        stage_buf = [torch.empty(in_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        stage = [packed_views(sb, spec, in_offs) for sb in stage_buf]
        out_buf = [torch.empty(out_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        outs_e = [[v["o"] for v in packed_views(ob, out_spec, out_offs)] for ob in out_buf]
        out_host = [torch.empty(out_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]

        def upload(t, b):
            stage_buf[b].copy_(host_pk[t], non_blocking=True)

        def download(b):
            out_host[b].copy_(out_buf[b], non_blocking=True)
    else:
        pin = lambda t: None if t is None else t.cpu().pin_memory()
        host_dev = [[{k: pin(v) for k, v in x.items()} for x in per_layer] for per_layer in setup.dev]
        h2d = sum(v.numel() * v.element_size() for x in host_dev[0] for v in x.values() if v is not None)
        d2h = sum(o.numel() * o.element_size() for o in outs)
        stage = [[{k: (None if v is None else torch.empty_like(v)) for k, v in x.items()}
                  for x in setup.dev[0]] for _ in range(2)]
        outs_e = [[torch.empty_like(o) for o in outs] for _ in range(2)]
        out_host = [[torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs] for _ in range(2)]

        def upload(t, b):
            for l in range(wl.n_layers):
                for k, v in host_dev[t][l].items():
                    if v is not None:
                        stage[b][l][k].copy_(v, non_blocking=True)

        def download(b):
            for l in range(wl.n_layers):
                out_host[b][l].copy_(outs_e[b][l], non_blocking=True)
    prep_2 = [[[dl.PreparedStep("decode", r.pool, l, gs, s_["q"], s_["k"], s_["v"], s_["lam"],
                                s_["beta"], outs_e[b][l], wl.lambda_const, auto_merge=r.merge)
                for l, s_ in enumerate(stage[b])]
               for b in range(2)] for gs in r.group_slots]
    copies = ("one H2D copy of the step's packed pinned inputs" if a.e2e_copies == "packed"
              else "H2D copies of the step's pinned inputs")
    copies_out = "one D2H copy of every layer's o_t" if a.e2e_copies == "packed" else "D2H of o_t"
    ndist = setup.ndist
    # the deferred leg ran W + K steps on every group before this leg
    j0 = W + K

    def serial_calls(j):
        j = j + j0
        t, prep = j % ndist, prep_2[j % R][0]

        def one():
            upload(t, 0)
            for p_ in prep:
                check_status(p_())
            download(0)
        return [one]

    # Pipelined: uploads on one copy stream, the decode calls on the current
    # stream, downloads on another copy stream, with buffer set j % 2 for step j.
    # Step j's upload waits until step j-2's kernels have read that set; its
    # kernels wait for its upload and for step j-2's download of the same
    # outputs; its download waits for its kernels.  So step j+1's upload and step
    # j-1's download run while step j computes.
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    last = W + K - 1

    def piped_calls(jl):
        j = jl + j0 + W + K
        t, b = j % ndist, jl % 2
        prep = prep_2[j % R][b]

        def one():
            comp = torch.cuda.current_stream()
            if jl == W:
                # the timed region starts at the compute stream's start event
                s_in.wait_stream(comp)
                s_out.wait_stream(comp)
            s_in.wait_event(ev_comp[b])
            with torch.cuda.stream(s_in):
                upload(t, b)
            ev_in[b].record(s_in)
            comp.wait_event(ev_in[b])
            comp.wait_event(ev_out[b])
            for p_ in prep:
                check_status(p_())
            ev_comp[b].record(comp)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                download(b)
            ev_out[b].record(s_out)
            if jl == last:
                comp.wait_stream(s_out)   # the end event follows the last download
        return [one]

    ms_s = ctx.timed(serial_calls, K, W, graph_ok=False)
    if r.errors() != 0:
        raise RuntimeError("device error bits set in the end-to-end leg")
    ctx.launches += K * wl.n_layers
    tot_s = ctx.reduce_max(ms_s)
    serial = {"value": whole_job_rate(wl.units_per_step * K, ctx.world, tot_s), "unit": UNIT,
              "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": tot_s / K,
              "copies": a.e2e_copies,
              "path": f"one stream: {copies} -> dl_decode_step per layer -> {copies_out}, "
                      "step after step, all inside the events"}
    if a.l2 != "rotate":
        return {"e2e": serial}
    ms_p = ctx.timed(piped_calls, K, W, graph_ok=False)
    if r.errors() != 0:
        raise RuntimeError("device error bits set in the end-to-end leg")
    ctx.launches += K * wl.n_layers
    tot_p = ctx.reduce_max(ms_p)
    e2e = {"value": whole_job_rate(wl.units_per_step * K, ctx.world, tot_p), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": tot_p / K,
           "copies": a.e2e_copies,
           "path": f"{copies} (copy stream) -> dl_decode_step per layer (compute "
                   f"stream) -> {copies_out} (second copy stream), double-buffered so "
                   "that step j+1's upload and step j-1's download overlap step j's "
                   "kernels; every copy inside the events"}
    return {"e2e": e2e, "e2e_serial": serial}


def run_gpu(a, wl, rank, world, dist):
    ctx = GpuContext(a, world, dist)
    K, W = a.steps, a.warmup
    rec, kept = measure_decode(ctx, wl, K, W, keep=not a.no_e2e)
    launches_headline = K * wl.n_layers
    result = {"value": rec["value"], "ms_per_step": rec["ms_per_step"], "roofline": rec["roofline"],
              "gpu_launches": launches_headline, "rotation_groups": rec["rotation_groups"],
              "live_entries": rec["live_entries"], "deferred_bytes_per_step": rec["deferred_bytes_per_step"],
              "merge_policy": rec["merge_policy"], "merges_every_step": rec["merges_every_step"]}
    for k in ("eager", "deferred_over_eager", "eager_bytes_over_deferred", "at_capacity"):
        if k in rec:
            result[k] = rec[k]
    if kept is not None:
        r, setup, R, goffs = kept
        result.update(measure_e2e(ctx, wl, K, W, r, setup, R, goffs))
        del r, setup, kept
        ctx.torch.cuda.empty_cache()
    subs = []
    for swl in spec_list(a.subs):
        Ks = sub_steps(swl, K, a.log_format)
        Ws = max(W, 3)
        from recurrent_state_serving_b200 import deltalog as dl
        if dl.dl_merge_policy(swl.batch, swl.n_heads, a.merge):
            # merging every step: a group's first step folds the log its staggering
            # pre-steps left; warm up one whole rotation so that the window is the
            # steady state (every slot starting empty)
            Ws = max(Ws, rotation_groups(swl, a.l2))
        srec, _ = measure_decode(ctx, swl, Ks, Ws)
        subs.append(srec)
    if subs:
        result["subs"] = subs
    merges = []
    for mwl in spec_list(a.merge_legs):
        merges.append(measure_merge(ctx, mwl, max(K, 4), max(W, 2)))
    if merges:
        result["merge_legs"] = merges
    result["gpu_launches_all_legs"] = ctx.launches
    result["graph_uploaded"] = ctx.graph_uploaded
    result["clocks"] = ctx.sampler.stop()
    return result


# ---------------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------------
def oracle_sample_rate(wl, target_s=10.0, threads=None):
    """fp64 eager oracle on the host cores over a bounded sample of the workload's
    heads (layer 0); returns (head-steps/s, threads, description).  Up to 64
    distinct seeded steps are generated and cycled to reach about target_s of
    oracle work; only the oracle call is timed.  threads: all host cores by default."""
    import oracle
    from recurrent_state_serving_b200 import synth
    threads = threads or os.cpu_count() or 1
    S0 = synth.initial_state(wl.with_(batch=min(wl.batch, 64)), 0).astype(np.float64)
    rows = np.arange(S0.shape[0])
    ndist = min(64, wl.steps)
    seq = [synth.select_rows(wl, synth.step_inputs(wl, t, 0), rows) for t in range(ndist)]
    f = lambda k, t: synth.input_to_f64(seq[t % ndist][k], wl.in_dtype)

    def run(T):
        Q = np.stack([f("q", t) for t in range(T)])
        Kk = np.stack([f("k", t) for t in range(T)])
        V = np.stack([f("v", t) for t in range(T)])
        LAM = None
        if wl.decay != "none":
            LAM = seq[0]["lam"].astype(np.float64) if wl.lambda_const else np.stack(
                [seq[t % ndist]["lam"].astype(np.float64) for t in range(T)])
        BETA = (np.stack([seq[t % ndist]["beta"].astype(np.float64) for t in range(T)])
                if wl.update == "delta" else None)
        t0 = time.perf_counter()
        oracle.eager_rollout(S0, Q, Kk, V, LAM, BETA, decay=wl.decay, update=wl.update,
                             lambda_const=wl.lambda_const, threads=threads)
        return time.perf_counter() - t0

    dt = run(8)
    heads = S0.shape[0] * wl.n_heads
    T = int(max(8, min(4096, 8 * target_s / max(dt, 1e-6))))
    dt = run(T)
    rate = heads * T / dt
    desc = (f"{heads} heads ({S0.shape[0]} slots x {wl.n_heads} heads, layer 0) x {T} steps of "
            f"{wl.name} ({ndist} distinct seeded steps cycled), fp64 eager oracle, {dt:.1f} s")
    return rate, threads, desc


def run_reference(a, wl):
    """Reference arm: the oracle, one bounded sample of the workload per step."""
    import oracle
    from recurrent_state_serving_b200 import synth
    threads = os.cpu_count() or 1
    budget_s = 90.0
    rows_all = np.arange(wl.batch)
    probe, _, _ = oracle_sample_rate(wl.with_(batch=min(wl.batch, 8)), target_s=1.0)
    per_step_heads = max(wl.n_heads, min(wl.units_per_step,
                                         int(probe * budget_s / max(1, a.steps + a.warmup))))
    n_rows = max(1, min(wl.batch, per_step_heads // wl.n_heads))
    rows = rows_all[:n_rows]
    S = synth.initial_state(wl.with_(batch=n_rows), 0).astype(np.float64)
    x = synth.step_inputs(wl, 0, 0)
    xs = synth.select_rows(wl, x, rows)
    f = lambda k: synth.input_to_f64(xs[k], wl.in_dtype)[None]
    Q, Kk, V = f("q"), f("k"), f("v")
    LAM = None
    if wl.decay != "none":
        LAM = xs["lam"].astype(np.float64) if wl.lambda_const else xs["lam"].astype(np.float64)[None]
    BETA = xs["beta"].astype(np.float64)[None] if wl.update == "delta" else None
    times = []
    for i in range(a.warmup + a.steps):
        t0 = time.perf_counter()
        _, Sck = oracle.eager_rollout(S, Q, Kk, V, LAM, BETA, decay=wl.decay, update=wl.update,
                                      lambda_const=wl.lambda_const, ckpts=[1], threads=threads)
        S = Sck[0]
        if i >= a.warmup:
            times.append(time.perf_counter() - t0)
    units = n_rows * wl.n_heads
    value = units * a.steps / sum(times)
    sample = (f"{units} of {wl.units_per_step} head-steps per step ({n_rows} slots x {wl.n_heads} heads, "
              f"layer 0), fp64 eager oracle advanced one token per step")
    # n_gpus echoes the launch (the arm is run with the same --gpus N as ours); the
    # oracle itself runs on the host cores of rank 0 and uses no GPU
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus,
            "device": f"host CPU, {threads} threads (no GPU)",
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * sum(times) / a.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl, 1, a.tile_v, a.l2, a.launch, a.log_format, a.replay,
                                                     a.phases),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    a = parse(argv)
    sys.path.insert(0, ROOT)
    wl = workload(a)
    if a.traffic_from:
        kern = {"decode": r"warp_head_kernel|step_kernel", "eager": r"step_kernel",
                "merge": r"merge_kernel|merge_head_kernel",
                "materialize": r"merge_kernel|merge_head_kernel"}[a.traffic_kind]
        text = traffic_summary_from_ncu(a.traffic_from, workload_key(wl, a.log_format), kern, a.traffic_kind)
        with open(PROFILE_TRAFFIC, "a") as f:
            f.write(text + "\n")
        print(text)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if a.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(a, wl)), flush=True)
        return

    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as td
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = td
    else:
        torch.cuda.set_device(0)

    res = run_gpu(a, wl, rank, world, dist)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded; bf16 q/k/v, fp32 lambda/beta, fp32 state and log)",
            "config": config_of(wl, world, a.tile_v, a.l2, a.launch, a.log_format, a.replay, a.phases),
            "roofline": res["roofline"], "gpu_launches": res["gpu_launches"],
            "hbm_tbs": res["roofline"]["achieved"] / 1e3}
    for k in ("live_entries", "merge_policy", "merges_every_step", "at_capacity", "eager",
              "deferred_over_eager", "eager_bytes_over_deferred",
              "deferred_bytes_per_step", "e2e", "e2e_serial", "clocks", "rotation_groups",
              "graph_uploaded", "subs", "merge_legs", "gpu_launches_all_legs"):
        if k in res:
            line[k] = res[k]
    if world == 1 and not a.no_cpu:
        rate, cores, desc = oracle_sample_rate(wl)
        rate1, _, desc1 = oracle_sample_rate(wl, target_s=3.0, threads=1)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": desc, "value_1core": rate1, "sample_1core": desc1}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
