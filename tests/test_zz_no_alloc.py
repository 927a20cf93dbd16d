"""GPU test of dl_decode_step_noalloc, the decode step for callers that cannot
allocate device memory (for example a serving engine that has already divided the
whole GPU among its own pools and refuses further cudaMalloc calls).  Instead of a
caller-provided arrival-counter buffer it uses a fixed device array inside the
library.  The test drives it through the C ABI side by side with dl_decode_step on
an identical pool and requires the same outputs, state, log and live lengths over
consecutive calls, merge steps included.

The file name sorts last so that a run that stops at the first failure has already
run every other test; it also passes on its own in a fresh process."""
import numpy as np
import pytest
import torch

from recurrent_state_serving_b200 import deltalog as dl
from recurrent_state_serving_b200 import synth
from recurrent_state_serving_b200.runner import DecodeRunner
from tests import harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("tile_v", [0, 16, 128])
def test_noalloc_step_matches_decode_step(tile_v):
    wl = synth.KDA.with_(n_layers=2, batch=5, n_heads=4, n_kheads=4, log_cap=4)
    ref = DecodeRunner(wl, n_slots=8, slot_seed=2, tile_v=tile_v)
    new = DecodeRunner(wl, n_slots=8, slot_seed=2, tile_v=tile_v)
    ref.load_initial_state()
    new.load_initial_state()
    new.pool.arrive.fill_(12345)   # must not be read or written by the allocation-free call
    for t in range(6):             # consecutive calls; step 4 is every slot's merge step
        for layer in range(wl.n_layers):
            x = ref.gen_inputs(t, layer)
            o_ref = ref.call(layer, x)
            o_new = dl.dl_decode_step_noalloc(new.pool, layer, new.slots, x["q"], x["k"], x["v"],
                                              lam=x["lam"], beta=x["beta"])
            H.check_steps(o_new.double().cpu().numpy()[None], o_ref.double().cpu().numpy()[None],
                          tol=H.REL_L2_GPU, elem=None, what=f"noalloc step {t} layer {layer}")
    torch.cuda.synchronize()
    assert ref.errors() == 0 and new.errors() == 0
    assert torch.equal(ref.pool.log_len, new.pool.log_len)
    assert H.rel_l2(new.pool.state.cpu().numpy(), ref.pool.state.cpu().numpy()) <= H.REL_L2_GPU
    assert H.rel_l2(new.pool.log.cpu().numpy(), ref.pool.log.cpu().numpy()) <= H.REL_L2_GPU
    assert int((new.pool.arrive != 12345).sum()) == 0


def test_noalloc_rejects_pools_beyond_its_counter_array():
    wl = synth.GLA_DIAG.with_(batch=2, n_heads=2, n_kheads=2, log_cap=4)
    r = DecodeRunner(wl)
    r.load_initial_state()
    x = r.gen_inputs(0, 0)
    desc = dl.dl_pool_desc.from_buffer_copy(r.pool.desc)
    desc.n_slots = 70000                      # 70000 slots x 1 layer > 65536 counters
    args = dl._step_args(r.pool, r.slots, x["q"], x["k"], x["v"], x["lam"], None,
                         torch.empty(2, 2, 128, device="cuda"), False)
    st = dl.library().dl_decode_step_noalloc(desc, 0, args, 1, None)
    assert st == dl.DL_ERR_SHAPE
