"""CPU tests of the algorithmic byte model against the figures the pages print."""
import json
import os

from recurrent_state_serving_b200 import synth, traffic

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "byte_model.json")


def test_byte_model_matches_printed_figures():
    fpga, paper = json.load(open(GOLDEN))["cases"]
    wl = synth.GDN_GVA.with_(n_heads=fpga["n_heads"], d_k=fpga["d"], d_v=fpga["d"])
    eager_state = wl.n_heads * (traffic.eager_head_step(wl) - traffic.token_bytes(wl))
    assert eager_state == fpga["state_io_bytes_per_token"]
    wl = synth.KDA.with_(batch=paper["batch"], n_heads=paper["n_heads"], d_k=paper["d"], d_v=paper["d"])
    assert wl.batch * wl.n_heads * traffic.state_bytes(wl) == paper["state_bytes"]
    assert wl.batch * wl.n_heads * 2 * traffic.state_bytes(wl) == paper["eager_state_traffic_bytes"]


def test_deferred_moves_fewer_bytes_than_eager_at_the_workload_intervals():
    for wl in (synth.GLA_DIAG, synth.GDN_GVA, synth.KDA, synth.RETNET):
        assert traffic.deferred_cycle_average(wl) < traffic.eager_head_step(wl)
    for L in synth.GLA_LOG_CAPS:
        wl = synth.GLA_DIAG.with_(log_cap=L)
        assert traffic.deferred_cycle_average(wl) < 0.75 * traffic.eager_head_step(wl)


def test_entry_and_token_sizes():
    assert traffic.entry_bytes(synth.KDA) == 1536
    assert traffic.entry_bytes(synth.GDN_GVA) == 1028
    assert traffic.entry_bytes(synth.TINY_LA) == 128
    # GVA: q and k shared by two value heads
    assert traffic.token_bytes(synth.GDN_GVA) == 2 * 128 * 2 / 2 + 256 + 4 + 4 + 512
    assert traffic.deferred_head_step(synth.KDA, 0, True) == traffic.eager_head_step(synth.KDA)


def test_compact_entry_bytes_agree_with_the_library_layout():
    """The byte model's compact entry (the bytes that must move) against the library's
    row size (dl_log_bytes): equal, except that scalar decay pads Lambda_0 to 16 B."""
    import ctypes
    from recurrent_state_serving_b200 import deltalog as dl
    for decay in ("none", "scalar", "diag"):
        for update in ("add", "delta"):
            wl = synth.GLA_DIAG.with_(decay=decay, update=update)
            d = dl.dl_pool_desc(1, 1, 1, 1, wl.d_k, wl.d_v, 1, dl.DECAY[decay], dl.UPDATE[update], 0,
                                dl.LOG_FORMAT["compact"], 0)
            n = ctypes.c_int64()
            assert dl.library().dl_log_bytes(ctypes.byref(d), ctypes.byref(n)) == dl.DL_OK
            pad = 12 if decay == "scalar" else 0
            assert traffic.entry_bytes(wl, "compact") + pad == n.value
            assert traffic.entry_bytes(wl, "compact") < traffic.entry_bytes(wl)
