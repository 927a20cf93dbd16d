"""CPU tests of the benchmark's bookkeeping: the ncu traffic summary it reads back,
and the byte accounting of the timed launches."""
import os

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
