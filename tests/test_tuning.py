"""Merge-interval selection: the byte model's U-curve and the pick from measurements."""
import math

import pytest

from recurrent_state_serving_b200 import synth, traffic, tuning

WLS = [synth.GLA_DIAG, synth.KDA, synth.RETNET, synth.GDN_GVA]


@pytest.mark.parametrize("wl", WLS, ids=lambda w: w.name)
@pytest.mark.parametrize("fmt", ["fp32", "compact"])
def test_interval_one_is_the_eager_step(wl, fmt):
    # L = 1: every step merges with an empty log, which is the eager recurrence
    assert tuning.cycle_bytes(wl, 1, fmt) == traffic.eager_head_step(wl)


@pytest.mark.parametrize("wl", WLS, ids=lambda w: w.name)
@pytest.mark.parametrize("fmt", ["fp32", "compact"])
def test_integer_minimum_brackets_the_real_optimum(wl, fmt):
    # the byte model is convex in L; its integer argmin over 1..256 is the floor or
    # the ceiling of sqrt(2 (S - e) / e)
    xs = range(1, 257)
    best = min(xs, key=lambda L: tuning.cycle_bytes(wl, L, fmt))
    lstar = tuning.continuous_optimum(wl, fmt)
    assert best in (math.floor(lstar), math.ceil(lstar))
    vals = [tuning.cycle_bytes(wl, L, fmt) for L in xs]
    diffs = [b - a for a, b in zip(vals, vals[1:])]
    # decreasing, then non-decreasing
    k = next(i for i, d in enumerate(diffs) if d >= 0)
    assert all(d < 0 for d in diffs[:k]) and all(d >= 0 for d in diffs[k:])


def test_real_optimum_of_a_hand_worked_case():
    # d = 128, per-key decay, fp32 log: S = 65536 B, e = 1536 B,
    # sqrt(2 * 64000 / 1536) = sqrt(83.33) = 9.129
    assert tuning.continuous_optimum(synth.GLA_DIAG) == pytest.approx(9.1287, abs=1e-4)
    # scalar decay: e = 1028 B -> sqrt(2 * 64508 / 1028) = 11.2028
    assert tuning.continuous_optimum(synth.RETNET) == pytest.approx(11.2028, abs=1e-4)


def test_modelled_pick_per_operator():
    c = (2, 4, 8, 16, 32, 64)
    assert tuning.modelled_log_cap(synth.GLA_DIAG, c) == 8
    assert tuning.modelled_log_cap(synth.RETNET, c) == 8
    # half-width entries move the optimum to a longer interval
    assert tuning.modelled_log_cap(synth.RETNET, c, "compact") == 16
    # a single candidate is its own pick; order and duplicates do not matter
    assert tuning.modelled_log_cap(synth.GLA_DIAG, (32,)) == 32
    assert tuning.modelled_log_cap(synth.GLA_DIAG, (64, 8, 8, 4)) == 8


def test_modelled_pick_agrees_with_the_measured_sweep():
    # GLA/RWKV6 diag, B = 64, H = 16, d = 128: decode head-steps/s measured on one
    # B200 for L in {4, 8, 16, 32} (inputs larger than L2, CUDA graph replay)
    measured = {4: 52.9e6, 8: 57.7e6, 16: 54.1e6, 32: 51.0e6}
    assert tuning.select_log_cap(measured) == 8
    assert tuning.modelled_log_cap(synth.GLA_DIAG, measured) == 8


def test_modelled_pick_agrees_with_the_retnet_sweep():
    # RetNet scalar decay, 8 layers, B = 256, H = 32, staggered merges: decode
    # head-steps/s on one B200 per interval and log layout (CUDA graph of 512 steps)
    fp32 = {8: 71.36e6, 16: 71.61e6, 32: 65.46e6}
    compact = {8: 72.77e6, 16: 75.86e6, 32: 71.76e6}
    wl = synth.RETNET.with_(batch=256)
    assert tuning.modelled_log_cap(wl, compact, "compact") == tuning.select_log_cap(compact) == 16
    # fp32: the model has L = 8 and 16 within 0.1 % of each other; so do the measurements
    assert tuning.modelled_log_cap(wl, fp32) == 8
    assert abs(fp32[8] / fp32[16] - 1) < 0.005
    assert tuning.cycle_bytes(wl, 16) / tuning.cycle_bytes(wl, 8) - 1 < 0.002


def test_select_from_measurements():
    assert tuning.select_log_cap({4: 1.0, 8: 3.0, 16: 2.0}) == 8
    # times: lower is better
    assert tuning.select_log_cap({4: 1.0, 8: 3.0, 16: 2.0}, higher_is_better=False) == 4
    # ties go to the smaller interval
    assert tuning.select_log_cap({16: 2.0, 8: 2.0, 32: 1.0}) == 8
    # unmeasured candidates are skipped
    assert tuning.select_log_cap({4: None, 8: float("nan"), 16: 0.5}) == 16
    with pytest.raises(ValueError):
        tuning.select_log_cap({4: None})
    with pytest.raises(ValueError):
        tuning.select_log_cap({0: 1.0})


def test_bad_arguments():
    with pytest.raises(ValueError):
        tuning.cycle_bytes(synth.GLA_DIAG, 0)
    with pytest.raises(ValueError):
        tuning.modelled_log_cap(synth.GLA_DIAG, ())
    with pytest.raises(ValueError):
        # d = 2 with per-key decay: an entry (24 B) outweighs the state (16 B)
        tuning.continuous_optimum(synth.GLA_DIAG.with_(d_k=2, d_v=2))


def test_sweep_table_and_cli(capsys):
    rows = tuning.sweep_table(synth.GLA_DIAG, (1, 8))
    assert rows[0][0] == 1 and rows[0][2] == pytest.approx(1.0)
    assert rows[1][2] < 1.0
    tuning.main(["--workload", "retnet_scalar", "--log-format", "compact", "--candidates", "8,16,32"])
    out = capsys.readouterr().out
    assert "modelled best L = 16" in out


def test_operator_pick_from_its_shape():
    assert tuning.auto_log_cap(128, 128, "diag", "add") == 8
    assert tuning.auto_log_cap(128, 128, "scalar", "add", "compact") == 16
    # the delta rule keeps b in fp32 in the compact layout: entry 772 B, optimum 12.9
    assert tuning.auto_log_cap(128, 128, "scalar", "delta", "compact", (8, 16)) == 16
    # no decay: no Lambda in the entry
    assert tuning.auto_log_cap(64, 64, "none", "add") == 8


def test_server_takes_the_modelled_interval():
    # pool construction touches no device memory through the library, so the
    # server's sizing runs on the host
    from recurrent_state_serving_b200.serving import DecodeServer
    kw = dict(n_slots=2, n_layers=1, n_heads=2, d_k=128, d_v=128, decay="scalar", device="cpu",
              use_graphs=False)
    s = DecodeServer(log_cap="auto", log_format="compact", **kw)
    assert s.log_cap == 16 and s.pool.log_cap == 16 and s.pool.log.shape[3] == 16
    assert DecodeServer(log_cap=5, **kw).log_cap == 5


def test_pick_from_bench_lines(tmp_path, capsys):
    """bench.py lines of an interval sweep (as --log-cap L runs print them) give the
    measured best interval per workload and log layout; reference lines are ignored."""
    import json

    import bench
    lines = []
    for L, v in {4: 52.9e6, 8: 57.7e6, 16: 54.1e6, 32: 51.0e6}.items():
        wl = synth.GLA_DIAG.with_(log_cap=L)
        lines.append(json.dumps({"value": v, "higher_is_better": True, "n_gpus": 1,
                                 "config": bench.config_of(wl, 1)}))
    for L, v in {8: 72.77e6, 16: 75.86e6, 32: 71.76e6}.items():
        wl = synth.RETNET.with_(log_cap=L)
        lines.append(json.dumps({"value": v, "higher_is_better": True, "n_gpus": 1,
                                 "config": bench.config_of(wl, 1, log_format="compact")}))
    ref = synth.GLA_DIAG.with_(log_cap=4)
    lines.append(json.dumps({"impl": "reference", "value": 1e12, "n_gpus": 1,
                             "config": bench.config_of(ref, 1)}))
    picks = tuning.select_from_bench_lines(lines)
    assert len(picks) == 2
    gla = next(v for k, v in picks.items() if k.startswith("gla_rwkv6_diag_b64_h16_d128 [fp32"))
    ret = next(v for k, v in picks.items() if "retnet" in k and "[compact" in k)
    assert gla[0] == 8 and sorted(gla[1]) == [4, 8, 16, 32]
    assert ret[0] == 16
    # the same through the command line, from a file with other output mixed in
    f = tmp_path / "sweep.jsonl"
    f.write_text("some log line\n" + "\n".join(lines) + "\n")
    tuning.main(["--from-bench", str(f)])
    out = capsys.readouterr().out
    assert "measured best L = 8" in out and "measured best L = 16" in out
