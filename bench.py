#!/usr/bin/env python
"""Benchmark of the base + log recurrent-state decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--log-cap L] [--batch B]

A step is one decode step of the whole batch over all layers of the workload (one
library call per layer), with every slot advancing by one token; merges happen on
each slot's own merge step inside the same call.  Inputs are seeded synthetic
tensors resident in HBM before timing starts.

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
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "step_kernel_traffic.txt")
CSRC = os.path.join(ROOT, "recurrent_state_serving_b200", "csrc")


def kernel_source_hash() -> str:
    """Hash of the CUDA sources; a recorded ncu traffic figure is only valid for it."""
    h = hashlib.sha256()
    for f in sorted(os.listdir(CSRC)):
        h.update(f.encode())
        h.update(open(os.path.join(CSRC, f), "rb").read())
    return h.hexdigest()[:16]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2048)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gla_rwkv6_diag")
    ap.add_argument("--log-cap", type=int, default=None)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-eager", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--traffic-from", default=None,
                    help="write profiles/step_kernel_traffic.txt from an ncu csv and exit")
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
    return ap.parse_args()


def workload(a):
    from recurrent_state_serving_b200 import synth
    wl = synth.WORKLOADS[a.workload]
    if a.log_cap:
        wl = wl.with_(log_cap=a.log_cap)
    if a.batch:
        wl = wl.with_(batch=a.batch)
    return wl


def rotation_groups(wl, l2_mode: str) -> int:
    """Slot groups stepped in turn so that the base states of one rotation total at
    least ROTATE_MIN_BYTES (1 under the flush method, or when one step's are enough)."""
    if l2_mode == "flush":
        return 1
    step_state = wl.units_per_step * 4 * wl.d_k * wl.d_v
    return max(1, -(-ROTATE_MIN_BYTES // step_state))


def l2_description(wl, l2_mode: str, launch: str) -> str:
    if l2_mode == "flush":
        return ("flushed before every timed step, outside the timed interval: 256 MiB write, then "
                "256 MiB read of another buffer (evicts the dirty lines); per-step CUDA events")
    R = rotation_groups(wl, l2_mode)
    mib = R * wl.units_per_step * 4 * wl.d_k * wl.d_v / 2**20
    return (f"inputs larger than L2: {R} slot group(s) of the batch stepped in turn, {mib:.0f} MiB of "
            f"base state per rotation (L2 126 MB); timed steps back to back, "
            f"{'replayed from one CUDA graph' if launch == 'graph' else 'launched directly'}")


def config_of(wl, n_gpus, tile_v=0, l2_mode="rotate", launch="graph", log_format="fp32", replay="per_tile"):
    suffix = "" if log_format == "fp32" else f"_{log_format}log"
    return {"workload": f"{wl.name}_b{wl.batch}_h{wl.n_heads}_d{wl.d_k}_L{wl.log_cap}{suffix}",
            "tile_v": tile_v or "auto", "log_format": log_format, "replay": replay,
            "layers": wl.n_layers, "batch_per_gpu": wl.batch, "heads": wl.n_heads,
            "kheads": wl.n_kheads, "d_k": wl.d_k, "d_v": wl.d_v, "log_cap": wl.log_cap,
            "decay": wl.decay, "update": wl.update, "inputs": wl.in_dtype, "state": "fp32",
            "l2": l2_description(wl, l2_mode, launch),
            "parallelism": f"replicas x{n_gpus} (independent slots, no collective)"}


def traffic_summary_from_ncu(csv_path: str, workload_key: str, kernel_regex: str) -> str:
    """Text for profiles/step_kernel_traffic.txt from an ncu --csv export of
    dram__bytes_read.sum and dram__bytes_write.sum over consecutive launches of the
    hot kernel (a whole merge cycle of every slot group: rotation groups x log
    capacity launches, so the mix of append and merge launches matches the timed
    region).  Run: python bench.py --traffic-from <csv>."""
    import csv
    import re
    rows = list(csv.reader(open(csv_path)))
    i = [k for k, r in enumerate(rows) if "Kernel Name" in r][0]
    hdr = rows[i]
    kn, mn, mv = hdr.index("Kernel Name"), hdr.index("Metric Name"), hdr.index("Metric Value")
    mu = hdr.index("Metric Unit") if "Metric Unit" in hdr else None
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}
    per = {}
    idcol = hdr.index("ID") if "ID" in hdr else None
    for r in rows[i + 1:]:
        if len(r) <= mv or not re.search(kernel_regex, r[kn]):
            continue
        if r[mn] not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        v = float(r[mv].replace(",", "")) * scale.get(r[mu] if mu is not None else "byte", 1)
        key = r[idcol] if idcol is not None else len(per)
        per[key] = per.get(key, 0.0) + v
    vals = list(per.values())
    if not vals:
        raise SystemExit("no matching launches in " + csv_path)
    avg = sum(vals) / len(vals)
    return (f"# ncu dram__bytes_read.sum + dram__bytes_write.sum per launch of the hot kernel,\n"
            f"# averaged over {len(vals)} consecutive launches (a whole merge cycle of every\n"
            f"# slot group, so append and merge launches mix as in the timed region).\n"
            f"workload = {workload_key}\nkernel_sha = {kernel_source_hash()}\n"
            f"launches = {len(vals)}\ndram_bytes_per_launch = {avg:.0f}\n"
            f"min_launch_bytes = {min(vals):.0f}\nmax_launch_bytes = {max(vals):.0f}\n")


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy)"
    return 6650.0, "fallback (6.65 TB/s)"


def recorded_traffic(workload_key):
    """Per-launch DRAM bytes of the step kernel from a committed ncu summary, or None
    when the summary is missing or the kernel source changed since it was taken."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    kv = {}
    for line in open(PROFILE_TRAFFIC):
        if "=" in line and not line.lstrip().startswith("#"):
            k, v = line.split("=", 1)
            kv[k.strip()] = v.strip()
    if kv.get("kernel_sha") != kernel_source_hash() or kv.get("workload") != workload_key:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


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


def live_entries(offsets, step_index: int, n_groups: int, log_cap: int):
    """Live log entries each slot of the group stepped at global step ``step_index``
    holds when the step starts: that group has taken step_index // n_groups steps
    before it, after its staggering pre-steps."""
    return (offsets + step_index // n_groups) % log_cap


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


def run_gpu(a, wl, rank, world, dist):
    import torch
    from recurrent_state_serving_b200 import deltalog as dl
    from recurrent_state_serving_b200 import synth, traffic
    from recurrent_state_serving_b200.runner import DecodeRunner

    dev = torch.device("cuda", torch.cuda.current_device())
    if a.l2 == "flush":
        flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        torch.sum(flush_rd, dim=0, out=flush_sink)
    L, K, W = wl.log_cap, a.steps, a.warmup
    ndist = max(1, min(wl.steps, 256 // wl.n_layers))

    def barrier_sync():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def reduce_max(x):
        return max_over_ranks(x, dist, dev)

    host_inputs = [[synth.step_inputs(wl, t, l) for l in range(wl.n_layers)] for t in range(ndist)]
    sampler = ClockSampler(dev.index)
    sampler.start()

    R = rotation_groups(wl, a.l2)
    use_graph = a.l2 == "rotate" and a.launch == "graph"
    graph_info = {}

    def timed(calls_for_step, n_steps, graph_ok=True):
        """calls_for_step(j) -> callables issued for global step j (one per layer).
        Returns the timed interval in ms (sum of the per-step intervals when flushing)."""
        for j in range(W):
            for c in calls_for_step(j):
                c()
        barrier_sync()
        if a.l2 == "flush":
            t0 = time.time()
            evs = []
            for i in range(n_steps):
                flush_l2()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                for c in calls_for_step(W + i):
                    c()
                e1.record()
                evs.append((e0, e1))
            barrier_sync()
            sampler.mark(t0, time.time())
            return sum(e0.elapsed_time(e1) for e0, e1 in evs)
        g = None
        if use_graph and graph_ok:
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
            graph_info["uploaded"] = graph_upload(g, torch.cuda.current_stream())
            barrier_sync()
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
        barrier_sync()
        sampler.mark(t0, time.time())
        ms = e0.elapsed_time(e1)
        del g
        return ms

    # ---- deferred (the product path) ----
    r = DecodeRunner(wl, device=str(dev), tile_v=a.tile_v, n_groups=R, log_format=a.log_format,
                     replay=a.replay)
    r.load_initial_state()
    r.run_presteps()
    dev_inputs = [[r.device_inputs(x) for x in per_layer] for per_layer in host_inputs]
    outs = [torch.empty(wl.batch, wl.n_heads, wl.d_v, dtype=torch.float32, device=dev)
            for _ in range(wl.n_layers)]

    def check(st):
        if st != 0:
            raise dl.DeltaLogError(st, "dl_decode_step")

    def prepared_calls(kind, runner, cache):
        """Step j: group j mod R, step inputs j mod ndist (argument blocks built once)."""
        def calls(j):
            key = (j % R, j % ndist)
            if key not in cache:
                g, t = key
                cache[key] = [dl.PreparedStep(kind, runner.pool, l, runner.group_slots[g], x["q"], x["k"],
                                              x["v"], x["lam"], x["beta"], outs[l], wl.lambda_const)
                              for l, x in enumerate(dev_inputs[t])]
            return [(lambda p=p: check(p())) for p in cache[key]]
        return calls

    total_ms = timed(prepared_calls("decode", r, {}), K)
    assert r.errors() == 0, "device error bits set during the benchmark"
    max_ms = reduce_max(total_ms)
    value = whole_job_rate(wl.units_per_step * K, world, max_ms)

    # algorithmic bytes of the timed launches: each slot enters its step with the
    # live entries of its own auto-merge cycle of length L
    offs = synth.slot_offsets(wl)
    bytes_total = 0.0
    for i in range(K):
        c = live_entries(offs, W + i, R, L)
        per_slot = [traffic.deferred_head_step(wl, int(cb), merge=(cb == L - 1), log_format=a.log_format)
                    for cb in c]
        bytes_total += sum(per_slot) * wl.n_heads * wl.n_layers
    launches = K * wl.n_layers
    achieved_gbs = bytes_total / (total_ms / 1e3) / 1e9
    peak, peak_src = measured_peaks()
    key = config_of(wl, world, log_format=a.log_format)["workload"]
    dram = recorded_traffic(key)
    roof = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved_gbs / peak, 4), "peak_source": peak_src,
            "traffic": dram, "algorithmic_bytes_per_launch": round(bytes_total / launches),
            "kernel": res_kernel_name(wl, a.tile_v), "launches_timed": launches,
            "avg_launch_us": round(total_ms * 1e3 / launches, 3),
            "frac_of_8tbs_spec": round(achieved_gbs / 8000.0, 4)}

    result = {"value": value, "ms_per_step": max_ms / K, "roofline": roof, "gpu_launches": launches,
              "rotation_groups": R}
    if use_graph:
        result["graph_uploaded"] = graph_info.get("uploaded")

    # ---- eager comparison (same workload, full read-modify-write each step) ----
    if not a.no_eager:
        re_ = DecodeRunner(wl, device=str(dev), mode="eager", tile_v=a.tile_v, n_groups=R)
        re_.load_initial_state()
        ms_e = timed(prepared_calls("eager", re_, {}), K)
        assert re_.errors() == 0
        tot_e = reduce_max(ms_e)
        eb = traffic.eager_head_step(wl) * wl.units_per_step * K
        result["eager"] = {"value": whole_job_rate(wl.units_per_step * K, world, tot_e),
                           "ms_per_step": tot_e / K,
                           "algorithmic_bytes_per_step": round(eb / K),
                           "achieved_gbs": round(eb / (ms_e / 1e3) / 1e9, 1)}
        result["deferred_bytes_per_step"] = round(bytes_total / K)
        del re_
        torch.cuda.empty_cache()

    # ---- end to end through the public API with host buffers ----
    if not a.no_e2e:
        # Inputs and outputs are double-buffered (set j % 2 for step j); the serial
        # form uses set 0 only.  --e2e-copies packed lays each step's inputs (all
        # layers) out in one pinned host buffer and every layer's output in one device
        # buffer, so a step is one upload and one download; per_tensor copies each
        # input and output tensor on its own.
        if a.e2e_copies == "packed":
            spec = [{k: (None if v is None else (tuple(v.shape), v.dtype)) for k, v in x.items()}
                    for x in dev_inputs[0]]
            in_bytes, in_offs = pack_layout(spec)
            host_pk = []
            for per_layer in dev_inputs:
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
            host_dev = [[{k: pin(v) for k, v in x.items()} for x in per_layer] for per_layer in dev_inputs]
            h2d = sum(v.numel() * v.element_size() for x in host_dev[0] for v in x.values() if v is not None)
            d2h = sum(o.numel() * o.element_size() for o in outs)
            stage = [[{k: (None if v is None else torch.empty_like(v)) for k, v in x.items()}
                      for x in dev_inputs[0]] for _ in range(2)]
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
                                    s_["beta"], outs_e[b][l], wl.lambda_const) for l, s_ in enumerate(stage[b])]
                   for b in range(2)] for gs in r.group_slots]
        copies = ("one H2D copy of the step's packed pinned inputs" if a.e2e_copies == "packed"
                  else "H2D copies of the step's pinned inputs")
        copies_out = "one D2H copy of every layer's o_t" if a.e2e_copies == "packed" else "D2H of o_t"

        def serial_calls(j):
            t, prep = j % ndist, prep_2[j % R][0]

            def one():
                upload(t, 0)
                for p_ in prep:
                    check(p_())
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

        def piped_calls(j):
            t, b = j % ndist, j % 2
            prep = prep_2[j % R][b]

            def one():
                comp = torch.cuda.current_stream()
                if j == W:
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
                    check(p_())
                ev_comp[b].record(comp)
                s_out.wait_event(ev_comp[b])
                with torch.cuda.stream(s_out):
                    download(b)
                ev_out[b].record(s_out)
                if j == last:
                    comp.wait_stream(s_out)   # the end event follows the last download
            return [one]

        # the calls a user makes, launched directly (no graph)
        ms_s = timed(serial_calls, K, graph_ok=False)
        assert r.errors() == 0
        tot_s = reduce_max(ms_s)
        serial = {"value": whole_job_rate(wl.units_per_step * K, world, tot_s), "unit": UNIT,
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": tot_s / K,
                  "copies": a.e2e_copies,
                  "path": f"one stream: {copies} -> dl_decode_step per layer -> {copies_out}, "
                          "step after step, all inside the events"}
        if a.l2 == "rotate":
            ms_p = timed(piped_calls, K, graph_ok=False)
            assert r.errors() == 0
            tot_p = reduce_max(ms_p)
            result["e2e"] = {"value": whole_job_rate(wl.units_per_step * K, world, tot_p), "unit": UNIT,
                             "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": tot_p / K,
                             "copies": a.e2e_copies,
                             "path": f"{copies} (copy stream) -> dl_decode_step per layer (compute "
                                     f"stream) -> {copies_out} (second copy stream), double-buffered so "
                                     "that step j+1's upload and step j-1's download overlap step j's "
                                     "kernels; every copy inside the events"}
            result["e2e_serial"] = serial
        else:
            result["e2e"] = serial
    result["clocks"] = sampler.stop()
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
    S = synth.initial_state(wl, 0)[rows].astype(np.float64)
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
            "data": "synthetic", "config": config_of(wl, 1, a.tile_v, a.l2, a.launch, a.log_format, a.replay),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    a = parse()
    sys.path.insert(0, ROOT)
    wl = workload(a)
    if a.traffic_from:
        key = config_of(wl, 1, log_format=a.log_format)["workload"]
        text = traffic_summary_from_ncu(a.traffic_from, key, r"warp_head_kernel|step_kernel")
        open(PROFILE_TRAFFIC, "w").write(text)
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
            "config": config_of(wl, world, a.tile_v, a.l2, a.launch, a.log_format, a.replay), "roofline": res["roofline"],
            "gpu_launches": res["gpu_launches"],
            "hbm_tbs": res["roofline"]["achieved"] / 1e3}
    for k in ("eager", "deferred_bytes_per_step", "e2e", "e2e_serial", "clocks", "rotation_groups",
              "graph_uploaded"):
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
