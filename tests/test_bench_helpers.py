"""CPU tests of the benchmark's bookkeeping: the ncu traffic summary it reads back,
and the byte accounting of the timed launches."""
import os

import numpy as np
import pytest

import bench
from recurrent_state_serving_b200 import synth, traffic


def _ncu_csv(path, launches):
    lines = ['"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"']
    for i, (rd, wr) in enumerate(launches):
        name = "void dl::wh::warp_head_kernel<2, false, __nv_bfloat16>(dl::KParams)"
        lines.append(f'"{i}","{name}","dram__bytes_read.sum","Mbyte","{rd}"')
        lines.append(f'"{i}","{name}","dram__bytes_write.sum","Mbyte","{wr}"')
        lines.append(f'"{i}","{name}","gpu__time_duration.sum","us","20.5"')
    lines.append('"99","void at::native::reduce_kernel<512>()","dram__bytes_read.sum","Mbyte","999"')
    open(path, "w").write("\n".join(lines) + "\n")


def test_traffic_summary_averages_matching_launches(tmp_path):
    p = tmp_path / "t.csv"
    _ncu_csv(p, [(70.0, 2.0), (72.0, 2.0), (130.0, 66.0), (71.0, 1.0)])
    text = bench.traffic_summary_from_ncu(str(p), "wl_key", r"warp_head_kernel")
    kv = dict(l.split(" = ") for l in text.splitlines() if " = " in l)
    assert kv["workload"] == "wl_key"
    assert kv["kernel_sha"] == bench.kernel_source_hash()
    assert int(kv["launches"]) == 4
    assert float(kv["dram_bytes_per_launch"]) == pytest.approx((72 + 74 + 196 + 72) / 4 * 1e6)


def test_recorded_traffic_is_dropped_when_kernels_change(tmp_path, monkeypatch):
    p = tmp_path / "traffic.txt"
    p.write_text(f"workload = k\nkernel_sha = {bench.kernel_source_hash()}\ndram_bytes_per_launch = 123\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(p))
    assert bench.recorded_traffic("k") == 123.0
    assert bench.recorded_traffic("other") is None
    p.write_text("workload = k\nkernel_sha = 0000\ndram_bytes_per_launch = 123\n")
    assert bench.recorded_traffic("k") is None


def test_cycle_byte_accounting_matches_the_model():
    """Bytes the bench charges to L consecutive launches of one slot phase cycle."""
    wl = synth.GLA_DIAG
    L = wl.log_cap
    per_cycle = sum(traffic.deferred_head_step(wl, c, merge=(c == L - 1)) for c in range(L))
    assert per_cycle / L == pytest.approx(traffic.deferred_cycle_average(wl))
    # the merge step moves the state twice, an append step once
    assert traffic.deferred_head_step(wl, L - 1, True) - traffic.deferred_head_step(wl, L - 1, False) == \
        pytest.approx(4 * wl.d_k * wl.d_v - traffic.entry_bytes(wl))


def test_rotation_groups_cover_three_l2_sizes():
    """Rotation: the groups' base states total >= 384 MiB, and one group fewer would not."""
    for wl in (synth.GLA_DIAG, synth.GDN_GVA, synth.RETNET.with_(batch=1), synth.RETNET.with_(batch=16),
               synth.KDA):
        R = bench.rotation_groups(wl, "rotate")
        step = wl.units_per_step * traffic.state_bytes(wl)
        assert R * step >= bench.ROTATE_MIN_BYTES
        assert R == 1 or (R - 1) * step < bench.ROTATE_MIN_BYTES
        assert bench.rotation_groups(wl, "flush") == 1
    assert bench.rotation_groups(synth.GLA_DIAG, "rotate") == 6      # 64 MiB per step
    assert bench.rotation_groups(synth.GDN_GVA, "rotate") == 192     # 2 MiB per step
    assert bench.rotation_groups(synth.KDA, "rotate") == 1


def test_live_entries_follow_each_group_cycle():
    """Group g is stepped at j = g, g + R, ...; before step j it has taken j // R steps."""
    import numpy as np
    offs = np.array([0, 3, 7])
    L, R = 8, 3
    seen = {g: 0 for g in range(R)}
    for j in range(40):
        g = j % R
        np.testing.assert_array_equal(bench.live_entries(offs, j, R, L), (offs + seen[g]) % L)
        seen[g] += 1
    # one group: the plain per-step cycle
    np.testing.assert_array_equal(bench.live_entries(offs, 13, 1, L), (offs + 13) % L)


def _step_spec(wl):
    import torch
    bf = torch.bfloat16 if wl.in_dtype == "bf16" else torch.float32
    x = synth.step_inputs(wl.with_(batch=3), 0, 0)
    spec = []
    for _ in range(wl.n_layers):
        d = {}
        for k, v in x.items():
            d[k] = None if v is None else (tuple(v.shape), bf if k in ("q", "k", "v") else torch.float32)
        spec.append(d)
    return spec


@pytest.mark.parametrize("wl", [synth.GLA_DIAG, synth.KDA.with_(n_layers=3), synth.RETNET.with_(n_layers=2),
                                synth.GDN_GVA, synth.TINY_LA], ids=lambda w: w.name)
def test_packed_step_inputs(wl):
    """One buffer per step: every tensor on a 256-byte boundary, no overlaps, the
    views round-trip the values, and the binding takes them as they are."""
    import torch
    from recurrent_state_serving_b200 import deltalog as dl
    spec = _step_spec(wl)
    total, offs = bench.pack_layout(spec)
    assert total % bench.PACK_ALIGN == 0
    spans = []
    for layer, o in zip(spec, offs):
        for k, v in layer.items():
            if v is None:
                assert o[k] is None
                continue
            n = int(np.prod(v[0])) * bench.torch_elem_size(v[1])
            assert o[k] % bench.PACK_ALIGN == 0
            spans.append((o[k], o[k] + n))
    spans.sort()
    assert all(a1 <= b0 for (_, a1), (b0, _) in zip(spans, spans[1:]))
    assert spans[-1][1] <= total
    padding = total - sum(b - a for a, b in spans)
    assert 0 <= padding < bench.PACK_ALIGN * (len(spans) + 1)

    buf = torch.zeros(total, dtype=torch.uint8)
    views = bench.packed_views(buf, spec, offs)
    g = torch.Generator().manual_seed(5)
    vals = []
    for layer in views:
        d = {}
        for k, v in layer.items():
            if v is not None:
                assert v.is_contiguous() and v.data_ptr() % bench.PACK_ALIGN == buf.data_ptr() % bench.PACK_ALIGN
                d[k] = torch.randn(v.shape, generator=g).to(v.dtype)
                v.copy_(d[k])
        vals.append(d)
    again = bench.packed_views(buf.clone(), spec, offs)
    for d, layer in zip(vals, again):
        for k, v in d.items():
            assert torch.equal(layer[k], v)

    # the binding accepts the views and passes their own addresses (no copies)
    class _RC(torch.Tensor):
        @property
        def is_cuda(self):
            return True
    rc = lambda t: None if t is None else torch.Tensor._make_subclass(_RC, t)
    B = 3
    pool = dl.Pool(B, wl.n_layers, wl.n_heads, wl.d_k, wl.d_v, 4, decay=wl.decay, update=wl.update,
                   n_kheads=wl.n_kheads, device="cpu")
    out_spec = [{"o": ((B, wl.n_heads, wl.d_v), torch.float32)} for _ in range(wl.n_layers)]
    ob, oo = bench.pack_layout(out_spec)
    outs = bench.packed_views(torch.zeros(ob, dtype=torch.uint8), out_spec, oo)
    slots = rc(torch.arange(B, dtype=torch.int32))
    for layer, o in zip(views, outs):
        a = dl._step_args(pool, slots, rc(layer["q"]), rc(layer["k"]), rc(layer["v"]), rc(layer["lam"]),
                          rc(layer["beta"]), rc(o["o"]), wl.lambda_const)
        assert a.q == layer["q"].data_ptr() and a.v == layer["v"].data_ptr()
        assert a.out == o["o"].data_ptr()


def test_spread_phases_give_every_launch_the_cycle_average():
    """With spread phases a batch of L or more slots holds each live length equally in
    every launch, so any window of timed steps is the amortised step."""
    for wl in (synth.KDA, synth.GLA_DIAG, synth.RETNET.with_(batch=1024, staggered=False)):
        R = bench.rotation_groups(wl, "rotate")
        go = bench.phase_offsets(wl, R, "spread")
        assert go.shape == (R, wl.batch)
        L = wl.log_cap
        for first, K in ((0, 1), (5, 20), (3, 7)):
            b, hist = bench.timed_window_bytes(wl, go, first, K)
            assert (hist == hist[0]).all() and hist.sum() == K * wl.batch
            per = b / (K * wl.units_per_step)
            assert per == pytest.approx(traffic.deferred_cycle_average(wl))
        assert L - 1 in set(bench.group_live_entries(go, 0, L))


def test_spread_phases_continue_across_groups_for_small_batches():
    """Batch 1 (GDN): launch j holds live length (j + j // R) mod L, so consecutive
    launches walk the merge cycle and L of them cover it once."""
    wl = synth.GDN_GVA
    R = bench.rotation_groups(wl, "rotate")
    go = bench.phase_offsets(wl, R, "spread")
    L = wl.log_cap
    for j in range(3 * R):
        assert bench.group_live_entries(go, j, L)[0] == (j % R + j // R) % L
    _, hist = bench.timed_window_bytes(wl, go, 0, L)
    assert (hist == 1).all()


def test_staggered_workload_keeps_its_own_offsets_in_group_zero():
    wl = synth.RETNET.with_(batch=64)
    go = bench.phase_offsets(wl, 3, "spread")
    np.testing.assert_array_equal(go[0], synth.slot_offsets(wl))
    np.testing.assert_array_equal(go[1], (synth.slot_offsets(wl) + 64) % wl.log_cap)
    np.testing.assert_array_equal(bench.phase_offsets(wl, 3, "workload"), np.tile(synth.slot_offsets(wl), (3, 1)))
    # group_live_entries with equal offsets per group is the single-offset rule
    for j in range(20):
        np.testing.assert_array_equal(bench.group_live_entries(np.tile(synth.slot_offsets(wl), (3, 1)), j, 32),
                                      bench.live_entries(synth.slot_offsets(wl), j, 3, 32))


def test_sub_record_steps_and_specs():
    for spec in bench.DEFAULT_SUBS.split(","):
        wl = bench.parse_spec(spec)
        n = bench.sub_steps(wl, 20)
        assert n >= 20 and n % wl.log_cap == 0 and n <= bench.SUB_MAX_STEPS
    wl = bench.parse_spec("gla_rwkv6_diag:b64:L8")
    assert (wl.batch, wl.log_cap) == (64, 8)
    assert bench.parse_spec("retnet_scalar:b1024").batch == 1024
    assert bench.parse_spec("kda_diag_delta:n1:b32").n_layers == 1
    with pytest.raises(SystemExit):
        bench.parse_spec("nope")
    with pytest.raises(SystemExit):
        bench.parse_spec("kda_diag_delta:x3")
    assert bench.spec_list("none") == []
    assert bench.parse(["--steps", "20"]).workload == "kda_diag_delta"


def test_distinct_steps_bounds_host_generation():
    for wl in (synth.KDA, synth.RETNET.with_(batch=1024), synth.GLA_DIAG, synth.GDN_GVA):
        n = bench.distinct_steps(wl)
        assert 2 <= n <= max(2, wl.steps)
        assert n == 2 or n * traffic.token_bytes(wl) * wl.units_per_step <= bench.HOST_INPUT_BYTES


def test_config_names_the_delta_reading():
    cfg = bench.config_of(synth.KDA, 1)
    assert "decayed" in cfg["delta_reading"] and cfg["workload"] == "kda_diag_delta_b256_h32_d128_L16"
    assert "delta_reading" not in bench.config_of(synth.GLA_DIAG, 1)


def test_traffic_records_by_kind(tmp_path, monkeypatch):
    p = tmp_path / "t.txt"
    sha = bench.kernel_source_hash()
    p.write_text(f"workload = w\nkind = decode\nkernel_sha = {sha}\ndram_bytes_per_launch = 10\n\n"
                 f"workload = w\nkind = eager\nkernel_sha = {sha}\ndram_bytes_per_launch = 20\n"
                 f"l2_write_bytes_per_launch = 7\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(p))
    assert bench.recorded_traffic("w") == 10.0
    assert bench.recorded_traffic("w", "eager") == 20.0
    assert bench.recorded_traffic("w", "eager", "l2_write_bytes_per_launch") == 7.0
    assert bench.recorded_traffic("w", "merge") is None


def test_expected_live_lengths_follow_the_steps_taken():
    wl = synth.GLA_DIAG
    R = 6
    go = bench.phase_offsets(wl, R, "spread")
    for n in (0, 1, 5, 6, 7, 53):
        want = bench.expected_live_lengths(wl, go, n)
        for g in range(R):
            taken = len([j for j in range(n) if j % R == g])
            np.testing.assert_array_equal(want[g], (go[g] + taken) % wl.log_cap)
    # merging every step: stepped groups are empty, the others keep their offsets
    ev = bench.expected_live_lengths(wl, go, 4, merge_every=True)
    assert not ev[:4].any()
    np.testing.assert_array_equal(ev[4:], go[4:])


def test_merge_every_window_counts_each_groups_first_fold():
    """Under the adaptive policy a group's first step folds its pre-step entries (a
    merge with c > 0); its later steps start empty."""
    wl = synth.GDN_GVA
    R = bench.rotation_groups(wl, "rotate")
    go = bench.phase_offsets(wl, R, "spread")
    L = wl.log_cap
    b, hist = bench.timed_window_bytes(wl, go, 3, 10, merge_every=True)
    want = np.bincount(go[3:13, 0], minlength=L)
    np.testing.assert_array_equal(hist, want)
    per_c = [traffic.deferred_head_step(wl, c, merge=True) for c in range(L)]
    assert b == pytest.approx(float(np.dot(want, per_c)) * wl.n_heads * wl.n_layers)
    _, hist2 = bench.timed_window_bytes(wl, go, R, 5, merge_every=True)   # second round: empty
    assert hist2[0] == 5 and hist2[1:].sum() == 0


def test_reference_arm_prints_the_oracle_line():
    """bench.py --impl reference times the fp64 oracle on the host cores (no GPU) and
    prints one JSON line with the same metric, unit and config as the GPU arm."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    run = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", "gla_rwkv6_diag:b4", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=root)
    assert run.returncode == 0, run.stderr[-2000:]
    lines = [ln for ln in run.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["higher_is_better"] is True and d["dtype"] == "f64"
    assert d["config"]["workload"] == "gla_rwkv6_diag_b4_h16_d128_L8"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the reference arm runs and prints on rank 0 alone; any other rank
    exits 0 without work or output."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    run = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", "gla_rwkv6_diag:b4", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=root, env=env)
    assert run.returncode == 0, run.stderr[-2000:]
    assert not [ln for ln in run.stdout.splitlines() if ln.startswith("{")]
