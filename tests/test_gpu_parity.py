"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, and the
deferred path against the in-library eager path.  Needs a B200."""
import numpy as np
import pytest
import torch

from recurrent_state_serving_b200 import deltalog as dl
from recurrent_state_serving_b200 import synth
from recurrent_state_serving_b200.runner import DecodeRunner
from tests import harness as H

pytestmark = pytest.mark.gpu

# Reduced sizes: several heads and value tiles, odd batch sizes, non-contiguous slot
# ids in a larger pool, and 256 steps (so every log fill level and many merges occur).
REDUCED = {
    "tiny_la": synth.TINY_LA,
    "gla_L4": synth.GLA_DIAG.with_(batch=5, n_heads=3, n_kheads=3, log_cap=4),
    "gla_L8": synth.GLA_DIAG.with_(batch=5, n_heads=3, n_kheads=3, log_cap=8),
    "gla_L16": synth.GLA_DIAG.with_(batch=3, n_heads=3, n_kheads=3, log_cap=16),
    "gla_L32": synth.GLA_DIAG.with_(batch=3, n_heads=3, n_kheads=3, log_cap=32),
    "gdn_gva": synth.GDN_GVA,
    "gdn_gva_256": synth.GDN_GVA.with_(batch=3, steps=256),
    "kda": synth.KDA.with_(n_layers=2, batch=3, n_heads=4, n_kheads=4, steps=256),
    "retnet": synth.RETNET.with_(n_layers=2, batch=7, n_heads=4, n_kheads=4, steps=256),
    # 128 x 128 heads without decay (linear attention, DeltaNet)
    "la_d128": synth.TINY_LA.with_(batch=3, n_heads=3, n_kheads=3, d_k=128, d_v=128, steps=96,
                                   log_cap=12, qkv_std=1 / np.sqrt(128), init_std=0.02, in_dtype="bf16"),
    "deltanet_d128": synth.TINY_LA.with_(batch=3, n_heads=3, n_kheads=3, d_k=128, d_v=128, steps=96,
                                         log_cap=12, qkv_std=1 / np.sqrt(128), init_std=0.02,
                                         update="delta", k_l2norm=True, in_dtype="bf16"),
    # long logs: a merge of exactly 32 entries, and merges of more than 32 entries
    "kda_L33": synth.KDA.with_(n_layers=1, batch=3, n_heads=3, n_kheads=3, steps=140, log_cap=33),
    "gla_L64": synth.GLA_DIAG.with_(batch=2, n_heads=3, n_kheads=3, steps=200, log_cap=64,
                                    staggered=True),
    "retnet_L48": synth.RETNET.with_(n_layers=1, batch=3, n_heads=3, n_kheads=3, steps=160, log_cap=48),
    "kda_L40": synth.KDA.with_(n_layers=1, batch=2, n_heads=3, n_kheads=3, steps=128, log_cap=40,
                               staggered=True),
}


def _run_case(wl, update=None, slot_seed=0, extra_slots=3, tile_v=0, log_format="fp32"):
    T = wl.steps
    ck = sorted({0, 1, T // 2, T})
    r = DecodeRunner(wl, n_slots=wl.batch + extra_slots, slot_seed=slot_seed, update=update,
                     tile_v=tile_v, log_format=log_format)
    outs, states, _ = H.gpu_rollout(r, T, ckpts=ck)
    assert r.errors() == 0
    for layer in r.layers:
        O, S = H.oracle_reference(wl, layer, T, ckpts=ck, update=update)
        H.check_steps(outs[layer], O, what=f"{wl.name} layer {layer} output")
        H.check_steps(states[layer], S, elem=None, what=f"{wl.name} layer {layer} state")
    return r, outs


def _tile_ok(wl, tile_v):
    if tile_v == 32:
        return wl.d_k >= 64 and wl.d_v % 32 == 0
    if tile_v == 128:
        return wl.d_k == 128 and wl.d_v == 128
    return True


@pytest.mark.parametrize("tile_v", [16, 32, 128])
@pytest.mark.parametrize("name", sorted(REDUCED))
def test_parity_vs_oracle(name, tile_v):
    wl = REDUCED[name]
    if not _tile_ok(wl, tile_v):
        pytest.skip("tile width not applicable to this head shape")
    _run_case(wl, tile_v=tile_v)


@pytest.mark.parametrize("tile_v", [32, 128])
def test_parity_delta_undecayed_reading(tile_v):
    _run_case(synth.KDA.with_(n_layers=1, batch=3, n_heads=4, n_kheads=4, steps=96),
              update="delta_undecayed", tile_v=tile_v)
    _run_case(synth.GDN_GVA.with_(batch=2, steps=96), update="delta_undecayed", tile_v=tile_v)


@pytest.mark.parametrize("shape", [(64, 80), (64, 64), (128, 256), (16, 48), (128, 48)])
def test_parity_other_head_shapes(shape):
    dk, dv = shape
    wl = synth.KDA.with_(n_layers=1, batch=3, n_heads=4, n_kheads=2, d_k=dk, d_v=dv,
                         steps=40, log_cap=6, qkv_std=1 / np.sqrt(dk))
    tiles = [16, 32] if dk >= 64 and dv % 32 == 0 else [16]
    for tv in tiles:
        _run_case(wl, tile_v=tv)
        _run_case(synth.GLA_DIAG.with_(batch=3, n_heads=2, n_kheads=1, d_k=dk, d_v=dv, steps=40,
                                       log_cap=5, qkv_std=1 / np.sqrt(dk)), tile_v=tv)


@pytest.mark.parametrize("tiles", [(32, 16), (128, 128), (128, 32)])
@pytest.mark.parametrize("name", ["tiny_la", "gla_L8", "gla_L32", "gdn_gva_256", "kda", "retnet"])
def test_deferred_matches_eager_on_gpu(name, tiles):
    wl = REDUCED[name]
    T = wl.steps
    td, te = tiles
    if wl.d_k == 16:
        if tiles != (32, 16):
            pytest.skip("one tiling for d_k = 16")
        td = 16
    rd = DecodeRunner(wl, n_slots=wl.batch + 2, slot_seed=1, tile_v=td)
    re = DecodeRunner(wl, n_slots=wl.batch + 2, slot_seed=1, mode="eager", tile_v=te)
    od, sd, _ = H.gpu_rollout(rd, T, ckpts=[T])
    oe, se, _ = H.gpu_rollout(re, T, ckpts=[T])
    assert rd.errors() == 0 and re.errors() == 0
    for layer in rd.layers:
        H.check_steps(od[layer], oe[layer], tol=H.REL_L2_GPU, elem=None, what="deferred vs eager")
        H.check_steps(sd[layer], se[layer], tol=H.REL_L2_GPU, elem=None, what="state")


@pytest.mark.parametrize("tile_v", [0, 16, 128])
def test_log_cap_one_is_eager_bit_for_bit(tile_v):
    wl = synth.KDA.with_(n_layers=1, batch=4, n_heads=4, n_kheads=4, steps=24, log_cap=1)
    rd = DecodeRunner(wl, tile_v=tile_v)
    re = DecodeRunner(wl, mode="eager", tile_v=tile_v)
    od, sd, _ = H.gpu_rollout(rd, wl.steps, ckpts=[wl.steps])
    oe, se, _ = H.gpu_rollout(re, wl.steps, ckpts=[wl.steps])
    np.testing.assert_array_equal(od[0], oe[0])
    np.testing.assert_array_equal(sd[0], se[0])
    assert int(rd.pool.log_len.abs().sum()) == 0


@pytest.mark.parametrize("log_format", ["fp32", "compact"])
@pytest.mark.parametrize("tile_v", [16, 128])
def test_log_contents_match_the_deferred_oracle(tile_v, log_format):
    """Entry i of the ring holds (a_i, b_i, Lambda_i) exactly as the paper's log does."""
    from oracle.deferred import DeferredHead
    wl = synth.KDA.with_(n_layers=1, batch=2, n_heads=2, n_kheads=2, steps=11, log_cap=8)
    r = DecodeRunner(wl, tile_v=tile_v, log_format=log_format)
    _, _, inputs = H.gpu_rollout(r, wl.steps, keep_inputs=True)
    S0 = synth.initial_state(wl, 0)
    log = H.log_entries_f64(r.pool)
    live = r.pool.log_len.cpu().numpy()
    f = lambda x: synth.input_to_f64(x, wl.in_dtype)
    dk, dv = wl.d_k, wl.d_v
    for b in range(wl.batch):
        s = r.slot_ids[b]
        for h in range(wl.n_heads):
            ref = DeferredHead(S0[b, h], wl.log_cap, wl.decay, wl.update)
            for x in inputs[0]:
                ref.decode(f(x["q"][b, h]), f(x["k"][b, h]), f(x["v"][b, h]),
                           x["lam"][b, h], x["beta"][b, h])
            assert live[s, 0] == ref.live == 11 - 8
            for i in range(ref.live):
                ent = log[s, 0, h, i]
                np.testing.assert_allclose(ent[:dk], ref.K_log[i], rtol=0, atol=0)
                assert H.rel_l2(ent[dk:dk + dv], ref.U_log[i]) < 1e-5
                np.testing.assert_allclose(ent[dk + dv:], ref.Lam_log[i], rtol=1e-5, atol=1e-7)


MERGE_FLOW = {
    "kda": synth.KDA.with_(n_layers=1, batch=3, n_heads=4, n_kheads=4, steps=30, log_cap=5),
    "retnet": synth.RETNET.with_(n_layers=1, batch=3, n_heads=4, n_kheads=4, steps=30, log_cap=5,
                                 staggered=False),
    "la_d128": REDUCED["la_d128"].with_(steps=30, log_cap=5),
    "gla_L64": synth.GLA_DIAG.with_(batch=2, n_heads=3, n_kheads=3, steps=140, log_cap=64),
}


@pytest.mark.parametrize("log_format", ["fp32", "compact"])
@pytest.mark.parametrize("tile_v", [0, 16])
@pytest.mark.parametrize("name", sorted(MERGE_FLOW))
def test_append_then_merge_flow(name, tile_v, log_format):
    """dl_append fills all L rows, dl_merge folds them, decode continues; every state is
    read back with dl_materialize (whole-head merge kernel for tile_v 0, value-tiled
    for 16)."""
    wl = MERGE_FLOW[name]
    r = DecodeRunner(wl, n_slots=6, slot_seed=3, tile_v=tile_v, log_format=log_format)
    r.load_initial_state()
    T = wl.steps
    gpu_states = []
    for t in range(T):
        x = r.gen_inputs(t, 0)
        if t < 2 * wl.log_cap:   # append-only phase with explicit merges
            dl.dl_append(r.pool, 0, r.slots, x["q"], x["k"], x["v"], lam=x["lam"], beta=x["beta"],
                         lambda_per_head=wl.lambda_const)
            if (t + 1) % wl.log_cap == 0:
                assert int(r.pool.log_len[r.slots.long(), 0].min()) == wl.log_cap
                dl.dl_merge(r.pool, 0, r.slots)
        else:
            r.call(0, x)
        gpu_states.append(r.materialize(0).double().cpu().numpy())
    assert r.errors() == 0
    _, S = H.oracle_reference(wl, 0, T, ckpts=list(range(1, T + 1)))
    H.check_steps(np.stack(gpu_states), S, elem=None, what="state")


def test_materialize_leaves_pool_unchanged():
    wl = synth.GLA_DIAG.with_(batch=3, n_heads=2, n_kheads=2, steps=5, log_cap=8)
    r = DecodeRunner(wl)
    H.gpu_rollout(r, wl.steps)
    before = [t.clone() for t in (r.pool.state, r.pool.log, r.pool.log_len, r.pool.arrive)]
    r.materialize(0)
    torch.cuda.synchronize()
    for a, b in zip(before, (r.pool.state, r.pool.log, r.pool.log_len, r.pool.arrive)):
        assert torch.equal(a, b)


def test_empty_batch_is_a_noop():
    wl = synth.GLA_DIAG.with_(batch=2, n_heads=2, n_kheads=2, steps=1)
    r = DecodeRunner(wl)
    r.load_initial_state()
    snap = r.pool.state.clone()
    x = r.gen_inputs(0, 0)
    empty = torch.zeros(0, dtype=torch.int32, device="cuda")
    e = lambda t: t[:0].contiguous()
    out = dl.dl_decode_step(r.pool, 0, empty, e(x["q"]), e(x["k"]), e(x["v"]), lam=e(x["lam"]))
    dl.dl_merge(r.pool, 0, empty)
    dl.dl_reset_slots(r.pool, empty)
    assert out.shape == (0, 2, 128)
    assert torch.equal(snap, r.pool.state) and r.errors() == 0


@pytest.mark.parametrize("tile_v", [0, 128])
def test_out_of_range_slot_sets_error_and_spares_others(tile_v):
    wl = synth.GLA_DIAG.with_(batch=3, n_heads=2, n_kheads=2, steps=3, log_cap=4)
    good = DecodeRunner(wl, tile_v=tile_v)
    og, _, _ = H.gpu_rollout(good, wl.steps)
    bad = DecodeRunner(wl, tile_v=tile_v)
    bad.load_initial_state()
    slots = bad.slots.clone()
    slots[1] = 99
    outs = []
    for t in range(wl.steps):
        x = bad.gen_inputs(t, 0)
        outs.append(bad.call(0, x, slots=slots).double().cpu().numpy())
    assert bad.errors() & dl.DL_EBIT_SLOT_RANGE
    assert bad.errors() == 0          # cleared by the previous read
    o = np.stack(outs)
    np.testing.assert_array_equal(o[:, [0, 2]], og[0][:, [0, 2]])


@pytest.mark.parametrize("tile_v", [0, 128])
def test_eager_step_on_live_log_is_refused(tile_v):
    wl = synth.GLA_DIAG.with_(batch=2, n_heads=2, n_kheads=2, steps=2, log_cap=4)
    r = DecodeRunner(wl, tile_v=tile_v)
    H.gpu_rollout(r, 2)
    snap = r.pool.state.clone()
    x = r.gen_inputs(5, 0)
    dl.dl_eager_step(r.pool, 0, r.slots, x["q"], x["k"], x["v"], lam=x["lam"])
    assert r.errors() == dl.DL_EBIT_LIVE_LOG
    assert torch.equal(snap, r.pool.state)


@pytest.mark.parametrize("tile_v", [0, 128])
def test_full_log_without_auto_merge_is_refused(tile_v):
    wl = synth.GLA_DIAG.with_(batch=2, n_heads=2, n_kheads=2, steps=1, log_cap=3)
    r = DecodeRunner(wl, tile_v=tile_v)
    r.load_initial_state()
    for t in range(3):
        x = r.gen_inputs(t, 0)
        dl.dl_decode_step(r.pool, 0, r.slots, x["q"], x["k"], x["v"], lam=x["lam"], auto_merge=False)
    assert r.errors() == 0
    assert r.pool.log_len[r.slots.long(), 0].tolist() == [3, 3]
    snap = r.pool.log.clone()
    x = r.gen_inputs(3, 0)
    dl.dl_decode_step(r.pool, 0, r.slots, x["q"], x["k"], x["v"], lam=x["lam"], auto_merge=False)
    assert r.errors() == dl.DL_EBIT_LOG_FULL
    assert torch.equal(snap, r.pool.log)
    # with auto-merge the same call folds the full log and the token into the base
    o = dl.dl_decode_step(r.pool, 0, r.slots, x["q"], x["k"], x["v"], lam=x["lam"])
    assert r.errors() == 0 and r.pool.log_len[r.slots.long(), 0].tolist() == [0, 0]
    O, _ = H.oracle_reference(wl, 0, 4)
    H.check_steps(o.double().cpu().numpy()[None], O[3:4])


def test_reset_slots_empties_the_log_only():
    wl = synth.GLA_DIAG.with_(batch=3, n_heads=2, n_kheads=2, steps=3, log_cap=8)
    r = DecodeRunner(wl)
    H.gpu_rollout(r, 3)
    base = r.pool.state.clone()
    dl.dl_reset_slots(r.pool, r.slots[:2].contiguous())
    torch.cuda.synchronize()
    assert r.pool.log_len[r.slots.long(), 0].tolist() == [0, 0, 3]
    assert torch.equal(base, r.pool.state)
    dense = r.materialize(0)
    assert torch.equal(dense[0], base[r.slot_ids[0], 0])


@pytest.mark.parametrize("tile_v", [0, 128])
def test_lambda_per_head_diag_and_scalar(tile_v):
    for decay in ("scalar", "diag"):
        wl = synth.RETNET.with_(n_layers=1, batch=3, n_heads=4, n_kheads=4, steps=70, decay=decay,
                                staggered=False, log_cap=8)
        _run_case(wl, tile_v=tile_v)


# --------------------------------------------------------------------------------
# full sizes, in the launch configuration the benchmark times
# --------------------------------------------------------------------------------
@pytest.mark.parametrize("log_cap", synth.GLA_LOG_CAPS)
def test_fullsize_gla_all_heads(log_cap):
    wl = synth.GLA_DIAG.with_(log_cap=log_cap)
    r = DecodeRunner(wl)
    outs, states, _ = H.gpu_rollout(r, wl.steps, ckpts=[wl.steps])
    assert r.errors() == 0
    O, S = H.oracle_reference(wl, 0, wl.steps, ckpts=[wl.steps])
    H.check_steps(outs[0], O)
    H.check_steps(states[0], S, elem=None)


def test_fullsize_kda_sampled_rows():
    """KDA at full size (24 layers x 256 slots x 32 heads, L = 16, 64 steps): sampled
    rows of the first and last layer, outputs at every step and the logical state
    (dl_materialize) after step 32 and step 64."""
    wl = synth.KDA
    rows = np.array([0, 77, 160, 255])
    layers = [0, wl.n_layers - 1]
    ck = [wl.steps // 2, wl.steps]
    r = DecodeRunner(wl, layers=layers)
    outs, states, kept = H.gpu_rollout(r, wl.steps, ckpts=ck, keep_inputs=True, state_rows=rows,
                                       out_rows=rows)
    assert r.errors() == 0
    for l in layers:
        O, S = H.oracle_reference(wl, l, wl.steps, rows=rows, ckpts=ck, main_inputs=kept[l], main_selected=True)
        H.check_steps(outs[l], O)
        H.check_steps(states[l], S, elem=None, what=f"KDA layer {l} state")
    del r
    torch.cuda.empty_cache()


def test_fullsize_retnet_b256_every_layer_staggered():
    """RetNet as benchmarked: 8 layers x 256 slots x 32 heads, L = 32, staggered merge
    phases, 128 steps; sampled rows on every layer, outputs at every step and the
    logical state after the last step."""
    wl = synth.RETNET
    rows = np.array([3, 128, 250])
    T = wl.steps
    r = DecodeRunner(wl)
    outs, states, kept = H.gpu_rollout(r, T, ckpts=[T], keep_inputs=True, state_rows=rows, out_rows=rows)
    assert r.errors() == 0
    for l in r.layers:
        O, S = H.oracle_reference(wl, l, T, rows=rows, ckpts=[T], main_inputs=kept[l], main_selected=True)
        H.check_steps(outs[l], O, what=f"RetNet layer {l} output")
        H.check_steps(states[l], S, elem=None, what=f"RetNet layer {l} state")
    del r
    torch.cuda.empty_cache()


def test_more_heads_than_the_head_list_holds():
    """131,072 heads in one launch: each CTA has more heads than its head list holds
    (512 per CTA at 148 SMs), so heads are neither ordered nor split.  Staggered
    merges happen inside the window; sampled rows against the oracle."""
    wl = synth.RETNET.with_(n_layers=1, batch=4096, steps=12)
    rows = np.array([0, 2047, 4095])
    T = wl.steps
    r = DecodeRunner(wl, tile_v=128)
    outs, states, kept = H.gpu_rollout(r, T, ckpts=[T], keep_inputs=True, state_rows=rows, out_rows=rows)
    assert r.errors() == 0
    offs = synth.slot_offsets(wl)
    assert ((offs + T) >= wl.log_cap).any()   # some slots merge inside the window
    O, S = H.oracle_reference(wl, 0, T, rows=rows, ckpts=[T], main_inputs=kept[0], main_selected=True)
    H.check_steps(outs[0], O)
    H.check_steps(states[0], S, elem=None, what="state")
    del r
    torch.cuda.empty_cache()


def test_fullsize_retnet_b1024_sampled_rows():
    wl = synth.RETNET.with_(batch=1024)
    T = 40
    rows = np.array([1, 500, 1023])
    r = DecodeRunner(wl, layers=[3])
    outs, _, kept = H.gpu_rollout(r, T, keep_inputs=True)
    assert r.errors() == 0
    O, _ = H.oracle_reference(wl, 3, T, rows=rows, main_inputs=kept[3])
    H.check_steps(outs[3][:, rows], O)
    del r
    torch.cuda.empty_cache()


# ---- compact log layout (bf16 a_i, bf16 b_i without the delta rule) ----------------
COMPACT_CASES = [n for n in sorted(REDUCED) if REDUCED[n].in_dtype == "bf16"]


@pytest.mark.parametrize("tile_v", [16, 32, 128])
@pytest.mark.parametrize("name", COMPACT_CASES)
def test_compact_log_parity_vs_oracle(name, tile_v):
    wl = REDUCED[name]
    if not _tile_ok(wl, tile_v) or (tile_v == 32 and name not in ("gla_L8", "kda", "retnet", "gdn_gva")):
        pytest.skip("tile width not applicable (or covered by the other widths)")
    _run_case(wl, tile_v=tile_v, log_format="compact")


@pytest.mark.parametrize("tile_v", [16, 32, 128])
@pytest.mark.parametrize("name", ["gla_L8", "kda", "retnet", "gdn_gva_256", "deltanet_d128"])
def test_compact_log_matches_fp32_log(name, tile_v):
    """The compact layout stores the same values (bf16 inputs, exactly), so a compact
    pool computes what an fp32 pool does: bit for bit on the value-tiled kernels, whose
    order of summation is the same; within the GPU deferred tolerance on the whole-head
    kernel, whose stages hold a different number of entries per layout."""
    wl = REDUCED[name]
    if not _tile_ok(wl, tile_v):
        pytest.skip("tile width not applicable")
    T = min(wl.steps, 96)
    res = {}
    for fmt in ("fp32", "compact"):
        r = DecodeRunner(wl, n_slots=wl.batch + 1, slot_seed=2, tile_v=tile_v, log_format=fmt)
        res[fmt] = H.gpu_rollout(r, T, ckpts=[T])
        assert r.errors() == 0
    for layer in res["fp32"][0]:
        of, sf = res["fp32"][0][layer], res["fp32"][1][layer]
        oc, sc = res["compact"][0][layer], res["compact"][1][layer]
        if tile_v in (16, 32):
            np.testing.assert_array_equal(oc, of)
            np.testing.assert_array_equal(sc, sf)
        else:
            H.check_steps(oc, of, tol=H.REL_L2_GPU, elem=None, what="compact vs fp32 output")
            H.check_steps(sc, sf, tol=H.REL_L2_GPU, elem=None, what="compact vs fp32 state")


def test_compact_log_append_merge_and_materialize():
    """dl_append / dl_merge / dl_materialize read and write the compact layout."""
    wl = synth.GLA_DIAG.with_(batch=3, n_heads=3, n_kheads=3, steps=20, log_cap=6)
    out = {}
    for fmt in ("fp32", "compact"):
        r = DecodeRunner(wl, n_slots=4, slot_seed=5, log_format=fmt, tile_v=16)
        r.load_initial_state()
        seen = []
        for t in range(wl.steps):
            x = r.gen_inputs(t, 0)
            if t % 6 < 5:
                dl.dl_append(r.pool, 0, r.slots, x["q"], x["k"], x["v"], lam=x["lam"], beta=x["beta"])
            else:
                dl.dl_merge(r.pool, 0, r.slots)
            seen.append(r.materialize(0).double().cpu().numpy())
        assert r.errors() == 0
        out[fmt] = np.stack(seen)
    np.testing.assert_array_equal(out["compact"], out["fp32"])


def test_compact_log_refuses_fp32_inputs_on_gpu():
    wl = synth.TINY_LA.with_(d_k=128, d_v=128, n_heads=2, n_kheads=2, batch=2)
    r = DecodeRunner(wl, log_format="compact")
    r.load_initial_state()
    x = r.gen_inputs(0, 0)   # fp32 q/k/v
    with pytest.raises(dl.DeltaLogError) as e:
        r.call(0, x)
    assert e.value.status == dl.DL_ERR_DTYPE


# ---- ReplayPrep shared by a head's value tiles (cluster) vs formed by every tile ----
@pytest.mark.parametrize("tile_v", [16, 32])
@pytest.mark.parametrize("name", ["gla_L8", "kda", "retnet", "gdn_gva_256", "deltanet_d128", "kda_L33"])
def test_cluster_replay_matches_per_tile_bit_for_bit(name, tile_v):
    """The tiles of a cluster form the same coefficients the per-tile form does, with
    the same arithmetic, and read them from one another unchanged: results agree bit
    for bit (decode steps with merges; both log layouts' value-tiled kernels)."""
    wl = REDUCED[name]
    if not _tile_ok(wl, tile_v):
        pytest.skip("tile width not applicable")
    T = min(wl.steps, 80)
    res = {}
    for mode in ("cluster", "per_tile"):
        r = DecodeRunner(wl, n_slots=wl.batch + 1, slot_seed=4, tile_v=tile_v, replay=mode)
        res[mode] = H.gpu_rollout(r, T, ckpts=[T])
        assert r.errors() == 0
    for layer in res["cluster"][0]:
        np.testing.assert_array_equal(res["cluster"][0][layer], res["per_tile"][0][layer])
        np.testing.assert_array_equal(res["cluster"][1][layer], res["per_tile"][1][layer])


# ---- merge heads split into 2 or 4 parts (CTAs with fewer than 24 heads) ---------------
# (batch, heads, L): 3200 heads (21-22 per CTA, halves at c < 16); 2048 heads with
# L = 32 (13-14 per CTA, quarters); 1024 heads (6-7 per CTA, halves over the idle
# warps); 592 heads (4 per CTA, quarters); L = 17 (c = 16: quarters at 21-22 per CTA).
SPLIT_SHAPES = {"b200_h16_L4": (200, 16, 4), "b64_h32_L32": (64, 32, 32), "b64_h16_L8": (64, 16, 8),
                "b37_h16_L8": (37, 16, 8), "b200_h16_L17": (200, 16, 17)}


@pytest.mark.parametrize("shape", sorted(SPLIT_SHAPES))
@pytest.mark.parametrize("staggered,log_format", [(False, "fp32"), (True, "fp32"), (True, "compact")])
def test_split_merge_heads_match_the_oracle(shape, staggered, log_format):
    """Every CTA with fewer than 24 heads orders its heads and splits each merge without
    the delta rule into 2 or 4 row-range work items whose partial outputs combine in
    shared memory.  Non-staggered, every slot merges at once (every merge head is split,
    as far as the CTA's accumulators go); staggered, a few do."""
    B, Hh, L = SPLIT_SHAPES[shape]
    wl = synth.GLA_DIAG.with_(batch=B, n_heads=Hh, n_kheads=Hh, steps=L * 2 + 5, log_cap=L,
                              staggered=staggered)
    rows = np.array([0, B // 2 - 1, B - 1])
    r = DecodeRunner(wl, tile_v=128, log_format=log_format)
    T = wl.steps
    outs, states, kept = H.gpu_rollout(r, T, ckpts=[T], keep_inputs=True)
    assert r.errors() == 0
    O, S = H.oracle_reference(wl, 0, T, rows=rows, ckpts=[T], main_inputs=kept[0])
    H.check_steps(outs[0][:, rows], O)
    H.check_steps(states[0][:, rows], S, elem=None, what="state")
    # against the in-library eager step over every row
    re_ = DecodeRunner(wl, mode="eager", tile_v=16)
    oe, se, _ = H.gpu_rollout(re_, T, ckpts=[T])
    H.check_steps(outs[0], oe[0], tol=H.REL_L2_GPU, elem=None, what="deferred vs eager")
    H.check_steps(states[0], se[0], tol=H.REL_L2_GPU, elem=None, what="state")


@pytest.mark.parametrize("batch", [64, 128])
def test_split_heads_are_the_same_on_every_run(batch):
    """Two runs of the same staggered workload agree bit for bit (outputs, logs, live
    lengths, states): at seven heads per CTA (no head list) and at about fourteen
    (balanced schedule, merge heads split in two halves whose sum does not depend on
    which half ends first), whatever order the warps take their heads in."""
    wl = synth.GLA_DIAG.with_(batch=batch, n_heads=16, n_kheads=16, steps=20, log_cap=8, staggered=True)
    res = []
    for _ in range(2):
        r = DecodeRunner(wl, tile_v=128)
        o, _, _ = H.gpu_rollout(r, wl.steps)
        assert r.errors() == 0
        res.append((torch.as_tensor(o[0]), r.pool.log.clone(), r.pool.log_len.clone(), r.pool.state.clone()))
    for a, b in zip(res[0], res[1]):
        assert torch.equal(a, b)


def test_expired_wait_sets_the_timeout_bit_and_the_pool_recovers():
    """A wait of the whole-head kernel made to run out (test hook: one warp waits, for
    at most 2 ms, on a barrier nothing completes, with its first bulk copies in
    flight) sets DL_EBIT_TIMEOUT; the kernel drains its own copies and returns, the
    context stays usable, and after a fresh prefill and reset the same pool matches
    the oracle again."""
    wl = synth.GLA_DIAG.with_(batch=16, n_heads=16, n_kheads=16, steps=12, log_cap=4)
    r = DecodeRunner(wl, tile_v=128)
    r.load_initial_state()
    dl.dl_debug_stall(2_000_000)
    try:
        for t in range(2 * wl.log_cap):   # append steps and merge steps
            r.call(0, r.gen_inputs(t, 0))
        bits = dl.dl_read_error(r.pool, clear=False)
    finally:
        dl.dl_debug_stall(0)
    assert bits & dl.DL_EBIT_TIMEOUT, f"error bits {bits:#x}"
    assert dl.dl_read_error(r.pool, clear=True) == bits      # read, then cleared
    assert dl.dl_read_error(r.pool) == 0
    # ordinary calls on the same pool after prefill and reset
    T = wl.steps
    outs, states, _ = H.gpu_rollout(r, T, ckpts=[T])
    assert r.errors() == 0
    O, S = H.oracle_reference(wl, 0, T, ckpts=[T])
    H.check_steps(outs[0], O, what="output after recovery")
    H.check_steps(states[0], S, elem=None, what="state after recovery")


def test_read_error_clears_only_when_asked():
    wl = synth.GLA_DIAG.with_(batch=2, n_heads=2, n_kheads=2, steps=1)
    r = DecodeRunner(wl, n_slots=4)
    r.load_initial_state()
    x = r.gen_inputs(0, 0)
    bad = torch.tensor([0, 99], dtype=torch.int32, device="cuda")
    dl.dl_decode_step(r.pool, 0, bad, x["q"], x["k"], x["v"], lam=x["lam"])
    assert dl.dl_read_error(r.pool, clear=False) == dl.DL_EBIT_SLOT_RANGE
    assert dl.dl_read_error(r.pool, clear=False) == dl.DL_EBIT_SLOT_RANGE
    assert dl.dl_read_error(r.pool, clear=True) == dl.DL_EBIT_SLOT_RANGE
    assert dl.dl_read_error(r.pool, clear=False) == 0


@pytest.mark.parametrize("name", ["gdn_gva", "retnet", "kda"])
def test_adaptive_policy_matches_the_oracle(name):
    """DL_MERGE_ADAPTIVE on launches below a few heads per SM merges every slot on every
    step; switched on mid-run it first folds the live logs.  Outputs and states match
    the oracle under either policy, and the log stays empty once adaptive."""
    wl = REDUCED[name]
    assert dl.dl_merge_policy(wl.batch, wl.n_heads, "adaptive")
    T = 40
    half = 13
    r = DecodeRunner(wl, n_slots=wl.batch + 2, slot_seed=4, tile_v=0)
    r.load_initial_state()
    r.run_presteps()
    outs = {l: [] for l in r.layers}
    ck = {l: [] for l in r.layers}
    for t in range(T):
        r.merge = "capacity" if t < half else "adaptive"
        for l in r.layers:
            outs[l].append(r.call(l, r.gen_inputs(t, l)).double().cpu().numpy())
            if t + 1 in (half, T):
                ck[l].append(r.materialize(l).double().cpu().numpy())
        if t >= half:
            assert int(r.pool.log_len.abs().sum()) == 0
    assert r.errors() == 0
    for l in r.layers:
        O, S = H.oracle_reference(wl, l, T, ckpts=[half, T])
        H.check_steps(np.stack(outs[l]), O, what=f"{name} layer {l} output")
        H.check_steps(np.stack(ck[l]), S, elem=None, what=f"{name} layer {l} state")


def test_adaptive_policy_is_capacity_on_large_launches():
    """Above the threshold the adaptive policy is the at-capacity one: same outputs,
    same logs, bit for bit."""
    wl = synth.GLA_DIAG.with_(batch=64, n_heads=16, n_kheads=16, steps=12, log_cap=4)
    assert not dl.dl_merge_policy(wl.batch, wl.n_heads, "adaptive")
    res = []
    for merge in ("capacity", "adaptive"):
        r = DecodeRunner(wl, merge=merge)
        o, _, _ = H.gpu_rollout(r, wl.steps)
        res.append((o[0], r.pool.log.clone(), r.pool.log_len.clone(), r.pool.state.clone()))
    np.testing.assert_array_equal(res[0][0], res[1][0])
    for a, b in zip(res[0][1:], res[1][1:]):
        assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["kda_delta", "gla_add", "kda_compact"])
def test_mid_size_launches_match_the_oracle(name):
    """4096 heads (27-28 per CTA at 148 SMs, so per-CTA head lists with the merges
    first and no splits), staggered merges, delta and additive, both log layouts:
    every row against the oracle, and against the eager path."""
    base, fmt = {"kda_delta": (synth.KDA.with_(n_layers=1, batch=128, steps=24, log_cap=8, staggered=True), "fp32"),
                 "gla_add": (synth.GLA_DIAG.with_(batch=256, steps=24, log_cap=8, staggered=True), "fp32"),
                 "kda_compact": (synth.KDA.with_(n_layers=1, batch=128, steps=24, log_cap=8, staggered=True),
                                 "compact")}[name]
    wl = base
    T = wl.steps
    r = DecodeRunner(wl, tile_v=128, log_format=fmt)
    outs, states, _ = H.gpu_rollout(r, T, ckpts=[T])
    assert r.errors() == 0
    O, S = H.oracle_reference(wl, 0, T, ckpts=[T])
    H.check_steps(outs[0], O)
    H.check_steps(states[0], S, elem=None, what="state")
    # the logs agree with the eager path's states at the end, through dl_materialize
    re_ = DecodeRunner(wl, mode="eager", tile_v=16)
    oe, se, _ = H.gpu_rollout(re_, T, ckpts=[T])
    H.check_steps(outs[0], oe[0], tol=H.REL_L2_GPU, elem=None, what="deferred vs eager")
