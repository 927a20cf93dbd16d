"""CPU tests of the C ABI: the library loads, exports what the header declares, and
validates arguments on the host.  No call here reaches the GPU: every call either
fails validation or is a no-op (batch == 0) before any CUDA runtime call."""
import ctypes
import subprocess

import pytest
import torch

from recurrent_state_serving_b200 import deltalog as dl

EXPECTED = ["dl_append", "dl_create_pool", "dl_debug_stall", "dl_decode_step", "dl_decode_step_noalloc",
            "dl_destroy_pool", "dl_eager_step", "dl_log_bytes", "dl_materialize", "dl_merge", "dl_merge_policy",
            "dl_read_error", "dl_reset_slots", "dl_status_string"]


def test_header_declares_the_boundary():
    assert dl.header_functions() == EXPECTED


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(dl.LIB_PATH)
    for name in dl.header_functions():
        assert hasattr(lib, name), name


def test_only_the_abi_is_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", dl.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    text_syms = [l.split()[-1] for l in out.splitlines() if " T " in l]
    assert sorted(s for s in text_syms if s.startswith("dl_")) == EXPECTED
    assert not [s for s in text_syms if "dl" in s and not s.startswith("dl_")]


def _desc(**kw):
    base = dict(n_slots=4, n_layers=2, n_heads=4, n_kheads=2, d_k=128, d_v=128, log_cap=8,
                decay=2, update=1, tile_v=0, log_format=0, replay_mode=0, state=0x10000, log=0x20000, log_len=0x30000,
                arrive=0x40000, err_word=0x50000)
    base.update(kw)
    return dl.dl_pool_desc(**base)


def _create(desc):
    h = ctypes.c_void_p()
    st = dl.library().dl_create_pool(ctypes.byref(desc), ctypes.byref(h))
    return st, h


def test_create_pool_accepts_valid_descriptors():
    for kw in ({}, dict(d_k=16, d_v=16, n_kheads=4), dict(d_k=64, d_v=80), dict(log_cap=1),
               dict(log_cap=64), dict(log=None, log_len=None, arrive=None), dict(decay=0, update=0),
               dict(tile_v=16), dict(tile_v=32), dict(d_k=64, d_v=96, tile_v=32),
               dict(tile_v=128, log_cap=32), dict(tile_v=128, log_cap=64), dict(log_format=1),
               dict(log_format=1, decay=1, update=0, tile_v=128), dict(replay_mode=1)):
        st, h = _create(_desc(**kw))
        assert st == dl.DL_OK, (kw, dl.dl_status_string(st))
        assert dl.library().dl_destroy_pool(h) == dl.DL_OK


@pytest.mark.parametrize("kw,status", [
    (dict(n_slots=0), dl.DL_ERR_SHAPE),
    (dict(n_heads=6, n_kheads=4), dl.DL_ERR_SHAPE),
    (dict(d_k=32), dl.DL_ERR_SHAPE),
    (dict(d_k=100), dl.DL_ERR_SHAPE),
    (dict(d_v=40), dl.DL_ERR_SHAPE),
    (dict(d_v=2048), dl.DL_ERR_SHAPE),
    (dict(log_cap=0), dl.DL_ERR_SHAPE),
    (dict(log_cap=65), dl.DL_ERR_SHAPE),
    (dict(decay=3), dl.DL_ERR_INVALID_ARG),
    (dict(update=-1), dl.DL_ERR_INVALID_ARG),
    (dict(state=None), dl.DL_ERR_INVALID_ARG),
    (dict(state=0x10004), dl.DL_ERR_INVALID_ARG),
    (dict(err_word=None), dl.DL_ERR_INVALID_ARG),
    (dict(log_len=None), dl.DL_ERR_INVALID_ARG),
    (dict(arrive=None), dl.DL_ERR_INVALID_ARG),
    (dict(log=0x20008), dl.DL_ERR_INVALID_ARG),
    (dict(tile_v=8), dl.DL_ERR_SHAPE),
    (dict(tile_v=32, d_k=16, d_v=32), dl.DL_ERR_SHAPE),
    (dict(tile_v=32, d_v=80), dl.DL_ERR_SHAPE),
    (dict(tile_v=128, d_k=64, d_v=128), dl.DL_ERR_SHAPE),
    (dict(tile_v=128, d_v=256), dl.DL_ERR_SHAPE),
    (dict(tile_v=64), dl.DL_ERR_SHAPE),
    (dict(log_format=2), dl.DL_ERR_INVALID_ARG),
    (dict(log_format=-1), dl.DL_ERR_INVALID_ARG),
    (dict(replay_mode=2), dl.DL_ERR_INVALID_ARG),
])
def test_create_pool_rejects(kw, status):
    st, h = _create(_desc(**kw))
    assert st == status
    assert not h.value


def test_step_argument_validation_without_gpu():
    lib = dl.library()
    st, h = _create(_desc())
    assert st == dl.DL_OK
    P = 0x60000
    good = dict(slots=P, batch=2, q=P, k=P, v=P, in_dtype=1, lambda_=P, lambda_per_head=0,
                beta=P, out=P)

    def call(fn, **kw):
        a = dict(good)
        a.update(kw)
        args = dl.dl_step_args(**a)
        if fn == "dl_decode_step":
            return lib.dl_decode_step(h, 0, ctypes.byref(args), 1, None)
        return getattr(lib, fn)(h, 0, ctypes.byref(args), None)

    for fn in ("dl_decode_step", "dl_append", "dl_eager_step"):
        assert call(fn, batch=0) == dl.DL_OK                   # empty batch: no launch
        assert call(fn, batch=-1) == dl.DL_ERR_SHAPE
        assert call(fn, batch=5) == dl.DL_ERR_SHAPE            # more rows than slots
        assert call(fn, slots=None) == dl.DL_ERR_INVALID_ARG
        assert call(fn, q=None) == dl.DL_ERR_INVALID_ARG
        assert call(fn, in_dtype=7) == dl.DL_ERR_DTYPE
        assert call(fn, lambda_=None) == dl.DL_ERR_INVALID_ARG  # diag decay needs lambda
        assert call(fn, beta=None) == dl.DL_ERR_INVALID_ARG     # delta rule needs beta
        assert call(fn, lambda_per_head=2) == dl.DL_ERR_INVALID_ARG
        assert call(fn, q=P + 1) == dl.DL_ERR_INVALID_ARG       # misaligned bf16
    assert call("dl_decode_step", out=None) == dl.DL_ERR_INVALID_ARG
    assert call("dl_eager_step", out=None) == dl.DL_ERR_INVALID_ARG
    a = dl.dl_step_args(**good)
    assert lib.dl_decode_step(h, 2, ctypes.byref(a), 1, None) == dl.DL_ERR_INVALID_ARG  # layer
    assert lib.dl_decode_step(h, -1, ctypes.byref(a), 1, None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_decode_step(None, 0, ctypes.byref(a), 1, None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_merge(h, 0, P, 0, None) == dl.DL_OK
    assert lib.dl_merge(h, 0, None, 1, None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_merge(h, 3, P, 1, None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_materialize(h, 0, P, 1, None, None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_reset_slots(h, P, 0, None) == dl.DL_OK
    assert lib.dl_reset_slots(h, P, 9, None) == dl.DL_ERR_SHAPE
    assert lib.dl_read_error(h, None, 0, None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_destroy_pool(h) == dl.DL_OK
    assert lib.dl_destroy_pool(None) == dl.DL_ERR_INVALID_ARG


def test_eager_only_pool_rejects_log_operations():
    lib = dl.library()
    st, h = _create(_desc(log=None, log_len=None, arrive=None))
    P = 0x60000
    a = dl.dl_step_args(P, 1, P, P, P, 1, P, 0, P, P)
    assert lib.dl_decode_step(h, 0, ctypes.byref(a), 1, None) == dl.DL_ERR_UNSUPPORTED
    assert lib.dl_append(h, 0, ctypes.byref(a), None) == dl.DL_ERR_UNSUPPORTED
    assert lib.dl_merge(h, 0, P, 1, None) == dl.DL_ERR_UNSUPPORTED
    assert lib.dl_materialize(h, 0, P, 1, P, None) == dl.DL_ERR_UNSUPPORTED
    assert lib.dl_reset_slots(h, P, 1, None) == dl.DL_OK
    lib.dl_destroy_pool(h)


def test_status_strings():
    for s in range(7):
        assert dl.dl_status_string(s) and dl.dl_status_string(s) != "unknown status"
    assert dl.dl_status_string(99) == "unknown status"


def test_noalloc_entry_point_checks_without_gpu():
    """The allocation-free decode step validates its descriptor on the host (with the
    rules of dl_create_pool, minus the arrival buffer) before any CUDA call."""
    lib = dl.library()
    P = 0x60000
    a = dl.dl_step_args(P, 0, P, P, P, 1, P, 0, P, P)   # empty batch: no launch

    def call(**kw):
        d = _desc(**kw)
        return lib.dl_decode_step_noalloc(ctypes.byref(d), 0, ctypes.byref(a), 1, None)

    assert call(arrive=None) == dl.DL_OK
    assert call() == dl.DL_OK                           # a given arrive buffer is ignored
    assert call(arrive=None, log=None) == dl.DL_ERR_INVALID_ARG
    assert call(arrive=None, log_len=None) == dl.DL_ERR_INVALID_ARG
    assert call(arrive=None, d_k=100) == dl.DL_ERR_SHAPE
    assert call(arrive=None, n_slots=65536, n_layers=2) == dl.DL_ERR_SHAPE   # > 65536 counters
    assert call(arrive=None, n_slots=32768, n_layers=2) == dl.DL_OK
    assert lib.dl_decode_step_noalloc(None, 0, ctypes.byref(a), 1, None) == dl.DL_ERR_INVALID_ARG


def test_log_bytes_per_layout():
    """dl_log_bytes: rows x entry bytes of the layout (fp32 [a|b|Lambda], or compact with
    bf16 a, bf16 b without the delta rule, and Lambda per key / 4 floats / none)."""
    lib = dl.library()
    rows = 4 * 2 * 4 * 8

    def nbytes(**kw):
        n = ctypes.c_int64(-1)
        d = _desc(**kw)
        return lib.dl_log_bytes(ctypes.byref(d), ctypes.byref(n)), n.value

    for decay in (0, 1, 2):
        for update in (0, 1, 2):
            assert nbytes(decay=decay, update=update) == (dl.DL_OK, rows * 4 * (2 * 128 + 128))
    entry = {(0, 0): 512, (0, 1): 768, (1, 0): 528, (1, 1): 784, (2, 0): 1024, (2, 1): 1280}
    for (decay, update), e in entry.items():
        assert nbytes(decay=decay, update=update, log_format=1) == (dl.DL_OK, rows * e)
        assert e % 16 == 0
    assert nbytes(decay=2, update=2, log_format=1) == (dl.DL_OK, rows * 1280)
    assert nbytes(d_k=16, d_v=48, decay=1, update=0, log_format=1) == (dl.DL_OK, rows * (32 + 96 + 16))
    assert nbytes(log_format=3)[0] == dl.DL_ERR_INVALID_ARG
    assert nbytes(d_v=40)[0] == dl.DL_ERR_SHAPE
    assert lib.dl_log_bytes(None, None) == dl.DL_ERR_INVALID_ARG


def test_compact_log_needs_bf16_inputs():
    """A compact log stores k_t (and v_t) in bf16, exact only for bf16 inputs: decode and
    append steps with fp32 q/k/v are refused on the host."""
    lib = dl.library()
    st, h = _create(_desc(log_format=1))
    assert st == dl.DL_OK
    P = 0x60000
    a = dl.dl_step_args(P, 2, P, P, P, 0, P, 0, P, P)   # in_dtype = fp32
    assert lib.dl_decode_step(h, 0, ctypes.byref(a), 1, None) == dl.DL_ERR_DTYPE
    assert lib.dl_append(h, 0, ctypes.byref(a), None) == dl.DL_ERR_DTYPE
    d = _desc(log_format=1, arrive=None)
    assert lib.dl_decode_step_noalloc(ctypes.byref(d), 0, ctypes.byref(a), 1, None) == dl.DL_ERR_DTYPE
    lib.dl_destroy_pool(h)


class _ReportsCuda(torch.Tensor):
    """A host tensor that passes the binding's CUDA-tensor test, so that its later
    checks (device, shape) can be exercised without a GPU.  Every case below is
    refused before any library call."""
    @property
    def is_cuda(self):
        return True


def _rc(t):
    return torch.Tensor._make_subclass(_ReportsCuda, t)


def test_binding_checks_shapes_and_device_before_the_library():
    pool = dl.Pool(3, 1, 2, 16, 16, 4, decay="diag", update="delta", device="cpu")
    slots = _rc(torch.zeros(2, dtype=torch.int32))
    # materialize: the output buffer must be exactly [B, H, d_k, d_v]
    with pytest.raises(ValueError, match="dense_out must be"):
        dl.dl_materialize(pool, 0, slots, dense_out=_rc(torch.zeros(2, 2, 16, 17)))
    with pytest.raises(ValueError, match="dense_out must be"):
        dl.dl_materialize(pool, 0, slots, dense_out=_rc(torch.zeros(1, 2, 16, 16)))
    # tensors on another device than the pool's
    other = _rc(torch.zeros(2, dtype=torch.int32, device="meta"))
    for fn in (lambda s: dl.dl_materialize(pool, 0, s), lambda s: dl.dl_merge(pool, 0, s),
               lambda s: dl.dl_reset_slots(pool, s)):
        with pytest.raises(ValueError, match="is on meta"):
            fn(other)
    q = _rc(torch.zeros(2, 2, 16))
    v = _rc(torch.zeros(2, 2, 16))
    lam = _rc(torch.zeros(2, 2, 16))
    beta = _rc(torch.zeros(2, 2))
    out = _rc(torch.zeros(2, 2, 16))
    with pytest.raises(ValueError, match="is on meta"):
        dl.dl_decode_step(pool, 0, slots, q, q, v, lam=lam, beta=_rc(torch.zeros(2, 2, device="meta")),
                          out=out)
    with pytest.raises(ValueError, match="lambda must be"):
        dl.dl_decode_step(pool, 0, slots, q, q, v, lam=_rc(torch.zeros(2, 2)), beta=beta, out=out)
    with pytest.raises(ValueError, match="out must be"):
        dl.dl_decode_step(pool, 0, slots, q, q, v, lam=lam, beta=beta, out=_rc(torch.zeros(2, 2, 8)))
    with pytest.raises(TypeError, match="CUDA tensor"):
        dl.dl_decode_step(pool, 0, slots, torch.zeros(2, 2, 16), q, v, lam=lam, beta=beta, out=out)


def test_header_compiles_as_c99_and_matches_the_binding(tmp_path):
    """A plain C consumer of include/deltalog.h: it must build with a C compiler in
    strict mode, link against the library, get the documented results from the
    calls that need no GPU, and see the same struct layouts as the ctypes binding."""
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(dl.LIB_PATH)
    exe = str(tmp_path / "c_abi_consumer")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(root, "include"), os.path.join(root, "tests", "c_abi_consumer.c"),
                    "-o", exe, "-L", libdir, "-ldeltalog", f"-Wl,-rpath,{libdir}"], check=True)
    run = subprocess.run([exe], capture_output=True, text=True)
    assert run.returncode == 0, run.stdout + run.stderr
    seen = dict(line.rsplit(" ", 1) for line in run.stdout.splitlines() if " " in line)
    assert seen["sizeof.dl_pool_desc"] == str(ctypes.sizeof(dl.dl_pool_desc))
    assert seen["sizeof.dl_step_args"] == str(ctypes.sizeof(dl.dl_step_args))
    n = 0
    for key, off in seen.items():
        struct, _, field = key.partition(".")
        if struct in ("dl_pool_desc", "dl_step_args"):
            cls = getattr(dl, struct)
            assert getattr(cls, "lambda_" if field == "lambda" else field).offset == int(off), key
            n += 1
    assert n == 22
    assert run.stdout.strip().endswith("OK")


def test_merge_policy_without_gpu():
    """DL_MERGE_ADAPTIVE merges every step only below a few heads per SM (148 SMs
    assumed when no device is visible); other policies never do."""
    assert dl.dl_merge_policy(1, 32, "adaptive")            # 32 heads
    assert dl.dl_merge_policy(16, 32, "adaptive")           # 512 heads
    assert not dl.dl_merge_policy(64, 32, "adaptive")       # 2048 heads
    assert not dl.dl_merge_policy(256, 32, "adaptive")
    assert not dl.dl_merge_policy(1, 32, "capacity") and not dl.dl_merge_policy(1, 32, False)
    assert not dl.dl_merge_policy(0, 32, "adaptive")
    out = ctypes.c_int32(5)
    assert dl.library().dl_merge_policy(1, 0, 2, ctypes.byref(out)) == dl.DL_ERR_INVALID_ARG
    assert dl.library().dl_merge_policy(-1, 4, 2, ctypes.byref(out)) == dl.DL_ERR_INVALID_ARG
    assert dl.library().dl_merge_policy(1, 4, 2, None) == dl.DL_ERR_INVALID_ARG
    assert dl.merge_code(True) == 1 and dl.merge_code("adaptive") == 2 and dl.merge_code(0) == 0
