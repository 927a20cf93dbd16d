"""Serving loop: slot allocation (CPU) and, on the GPU, requests that arrive and leave
at different steps (slots reused, batch size changing, merges at every request's own
L-th step, one CUDA graph per batch size) checked against the fp64 eager oracle of
each request's own token sequence."""
import numpy as np
import pytest

from recurrent_state_serving_b200 import synth
from recurrent_state_serving_b200.serving import SlotAllocator


def test_slot_allocator_reuses_the_lowest_free_slot():
    a = SlotAllocator(4)
    assert [a.alloc() for _ in range(3)] == [0, 1, 2]
    a.free(1)
    assert a.n_free == 2 and a.used == [0, 2]
    assert a.alloc() == 1
    assert a.alloc() == 3
    with pytest.raises(RuntimeError):
        a.alloc()
    with pytest.raises(ValueError):
        a.free(7)
    a.free(0)
    with pytest.raises(ValueError):
        a.free(0)
    with pytest.raises(ValueError):
        SlotAllocator(0)


def _host_server(**kw):
    # the pool's buffers are host tensors here: only the host-side checks run
    import torch
    from recurrent_state_serving_b200.serving import DecodeServer
    args = dict(n_slots=3, n_layers=2, n_heads=4, n_kheads=2, d_k=16, d_v=16, log_cap=4,
                decay="diag", update="delta", device="cpu", use_graphs=False)
    args.update(kw)
    return DecodeServer(**args), torch


def test_server_rejects_a_bad_prefill_without_taking_a_slot():
    srv, torch = _host_server()
    with pytest.raises(ValueError):
        srv.admit(torch.zeros(2, 4, 16, 8))
    assert srv.alloc.n_free == 3 and srv.active == []


def test_server_checks_every_step_input():
    srv, torch = _host_server()
    B = 2

    def layer(**over):
        x = {"q": torch.zeros(B, 2, 16), "k": torch.zeros(B, 2, 16), "v": torch.zeros(B, 4, 16),
             "lam": torch.zeros(B, 4, 16), "beta": torch.zeros(B, 4)}
        x.update(over)
        return x

    srv._check_inputs([layer(), layer()], B)
    with pytest.raises(ValueError, match="layers"):
        srv._check_inputs([layer()], B)
    with pytest.raises(ValueError, match="'beta' is missing"):
        srv._check_inputs([layer(), layer(beta=None)], B)
    # a per-head row would broadcast over the batch: refused
    with pytest.raises(ValueError, match="'lam' must be"):
        srv._check_inputs([layer(lam=torch.zeros(4, 16)), layer()], B)
    with pytest.raises(ValueError, match="'v' must be"):
        srv._check_inputs([layer(v=torch.zeros(B + 1, 4, 16)), layer()], B)
    add, _ = _host_server(update="add", decay="none")
    with pytest.raises(ValueError, match="no 'beta'"):
        add._check_inputs([layer(lam=None), layer(lam=None)], B)
    add._check_inputs([layer(lam=None, beta=None), layer(lam=None, beta=None)], B)


# -- GPU: a request schedule over 30 steps ---------------------------------------
L_LAYERS, H, HK, D, LOG_CAP = 2, 4, 2, 128, 5
# (step, action, request index): admissions and retirements
SCHEDULE = {0: [("admit", 0), ("admit", 1), ("admit", 2)], 4: [("admit", 3)], 9: [("retire", 1)],
            10: [("admit", 4), ("admit", 5)], 17: [("retire", 0), ("retire", 3)], 18: [("admit", 6)],
            23: [("retire", 2)]}
T_TOTAL = 30


def _rng(r, t, l):
    return np.random.default_rng([7, r, t, l])


def _bf16(x):
    return synth.bf16_bits_to_f32(synth.to_bf16_bits(x)).astype(np.float64)


def _tokens(r, t, l):
    """One request's inputs at its step t, layer l (float64 values of bf16 / fp32)."""
    g = _rng(r, t, l)
    q = _bf16(g.standard_normal((HK, D)) / np.sqrt(D))
    kraw = g.standard_normal((HK, D))
    k = _bf16(kraw / np.linalg.norm(kraw, axis=-1, keepdims=True))
    v = _bf16(g.standard_normal((H, D)) / np.sqrt(D))
    x = g.standard_normal((H, D)) + 4.0
    lam = np.float32(np.where(x >= 0, -np.log1p(np.exp(-x)), x - np.log1p(np.exp(x)))).astype(np.float64)
    beta = np.float32(1.0 / (1.0 + np.exp(-g.standard_normal(H)))).astype(np.float64)
    return q, k, v, lam, beta


def _prefill(r):
    g = np.random.default_rng([11, r])
    return np.float32(g.standard_normal((L_LAYERS, H, D, D)) * 0.02)


@pytest.mark.gpu
@pytest.mark.parametrize("tile_v,log_format,log_cap,merge", [
    (0, "fp32", LOG_CAP, "capacity"), (128, "fp32", LOG_CAP, "capacity"),
    (0, "compact", LOG_CAP, "capacity"), (128, "compact", LOG_CAP, "capacity"),
    (0, "fp32", "auto", "capacity"), (128, "compact", "auto", "capacity"), (0, "fp32", LOG_CAP, "adaptive")])
def test_server_requests_match_the_oracle(tile_v, log_format, log_cap, merge):
    import torch
    from oracle import eager_tasks
    from recurrent_state_serving_b200 import tuning
    from recurrent_state_serving_b200.serving import DecodeServer
    from tests import harness as Hn
    srv = DecodeServer(n_slots=6, n_layers=L_LAYERS, n_heads=H, n_kheads=HK, d_k=D, d_v=D,
                       log_cap=log_cap, decay="diag", update="delta", log_format=log_format,
                       tile_v=tile_v, max_batch=5, merge=merge)
    if log_cap == "auto":
        # the modelled interval of this operator, which the schedule's requests outlive
        assert srv.log_cap == tuning.auto_log_cap(D, D, "diag", "delta", log_format)
        assert 1 < srv.log_cap < 20
    dev = srv.device
    rid_of, steps_of, outs = {}, {}, {}
    for t in range(T_TOTAL):
        for act, ri in SCHEDULE.get(t, []):
            if act == "admit":
                rid_of[ri] = srv.admit(torch.from_numpy(_prefill(ri)))
                steps_of[ri], outs[ri] = 0, []
            else:
                srv.retire(rid_of[ri])
        order = [ri for rid in srv.active for ri, x in rid_of.items() if x == rid]
        if not order:
            continue
        inputs = []
        for l in range(L_LAYERS):
            toks = [_tokens(ri, steps_of[ri], l) for ri in order]
            bf = lambda a: torch.from_numpy(np.float32(a)).to(dev).to(torch.bfloat16)
            f32 = lambda a: torch.from_numpy(np.float32(a)).to(dev)
            inputs.append({"q": bf(np.stack([x[0] for x in toks])), "k": bf(np.stack([x[1] for x in toks])),
                           "v": bf(np.stack([x[2] for x in toks])), "lam": f32(np.stack([x[3] for x in toks])),
                           "beta": f32(np.stack([x[4] for x in toks]))})
        res = srv.step(inputs)
        got = [o.double().cpu().numpy() for o in res]
        for row, ri in enumerate(order):
            outs[ri].append(np.stack([got[l][row] for l in range(L_LAYERS)]))
            steps_of[ri] += 1
    assert srv.errors() == 0
    assert len(srv._graphs) >= 3          # several batch sizes were captured
    for ri, seq in outs.items():
        T = len(seq)
        gpu = np.stack(seq)                # [T, layers, H, D]
        for l in range(L_LAYERS):
            toks = [_tokens(ri, t, l) for t in range(T)]
            S0 = _prefill(ri)[l].astype(np.float64)
            g = np.arange(H) // (H // HK)
            q = np.stack([np.stack([x[0][g[h]] for x in toks]) for h in range(H)])
            k = np.stack([np.stack([x[1][g[h]] for x in toks]) for h in range(H)])
            v = np.stack([np.stack([x[2][h] for x in toks]) for h in range(H)])
            lam = np.stack([np.stack([x[3][h] for x in toks]) for h in range(H)])
            beta = np.stack([np.stack([x[4][h] for x in toks]) for h in range(H)])
            ref, _ = eager_tasks(S0, q, k, v, lam, beta, decay="diag", update="delta")
            Hn.check_steps(gpu[:, l], ref.transpose(1, 0, 2), what=f"request {ri} layer {l}")
