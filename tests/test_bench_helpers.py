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
