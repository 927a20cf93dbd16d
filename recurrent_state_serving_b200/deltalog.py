"""Python binding of libdeltalog.so (argument marshalling only).

The functions carry the C ABI's names and take torch CUDA tensors; every step of
the decode path runs in the library's sm_100a kernels.  There is no fallback:
if the shared library is missing this module raises on import.

``Pool`` allocates the caller-owned device buffers a pool descriptor names
(torch does the allocation; the library allocates nothing) and owns the handle.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdeltalog.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "deltalog.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m recurrent_state_serving_b200.build` (nvcc, sm_100a)")
_lib = ctypes.CDLL(LIB_PATH)

DL_OK, DL_ERR_INVALID_ARG, DL_ERR_SHAPE, DL_ERR_DTYPE, DL_ERR_UNSUPPORTED, DL_ERR_CUDA, \
    DL_ERR_DEVICE = range(7)
DECAY = {"none": 0, "scalar": 1, "diag": 2}
UPDATE = {"add": 0, "delta": 1, "delta_undecayed": 2}
DTYPE = {torch.float32: 0, torch.bfloat16: 1}
LOG_FORMAT = {"fp32": 0, "compact": 1}
REPLAY = {"per_tile": 0, "cluster": 1}
DL_EBIT_SLOT_RANGE, DL_EBIT_LOG_FULL, DL_EBIT_LIVE_LOG, DL_EBIT_LOG_LEN, DL_EBIT_TIMEOUT = \
    0x1, 0x2, 0x4, 0x8, 0x10
DL_MERGE_NONE, DL_MERGE_AT_CAPACITY, DL_MERGE_ADAPTIVE = 0, 1, 2
MERGE = {False: DL_MERGE_NONE, True: DL_MERGE_AT_CAPACITY, "none": DL_MERGE_NONE,
         "capacity": DL_MERGE_AT_CAPACITY, "adaptive": DL_MERGE_ADAPTIVE}


def merge_code(auto_merge) -> int:
    """auto_merge as the C ABI's int: a bool, 'none' / 'capacity' / 'adaptive', or a DL_MERGE_* value."""
    if isinstance(auto_merge, (bool, str)):
        return MERGE[auto_merge]
    return int(auto_merge)


class dl_pool_desc(ctypes.Structure):
    _fields_ = [("n_slots", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("n_kheads", ctypes.c_int32),
                ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32), ("log_cap", ctypes.c_int32),
                ("decay", ctypes.c_int), ("update", ctypes.c_int), ("tile_v", ctypes.c_int32),
                ("log_format", ctypes.c_int32), ("replay_mode", ctypes.c_int32),
                ("state", ctypes.c_void_p), ("log", ctypes.c_void_p),
                ("log_len", ctypes.c_void_p), ("arrive", ctypes.c_void_p),
                ("err_word", ctypes.c_void_p)]


class dl_step_args(ctypes.Structure):
    _fields_ = [("slots", ctypes.c_void_p), ("batch", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("in_dtype", ctypes.c_int), ("lambda_", ctypes.c_void_p),
                ("lambda_per_head", ctypes.c_int32), ("beta", ctypes.c_void_p),
                ("out", ctypes.c_void_p)]


_vp = ctypes.c_void_p
_lib.dl_log_bytes.argtypes = [ctypes.POINTER(dl_pool_desc), ctypes.POINTER(ctypes.c_int64)]
_lib.dl_create_pool.argtypes = [ctypes.POINTER(dl_pool_desc), ctypes.POINTER(_vp)]
_lib.dl_destroy_pool.argtypes = [_vp]
_lib.dl_decode_step.argtypes = [_vp, ctypes.c_int32, ctypes.POINTER(dl_step_args), ctypes.c_int32, _vp]
_lib.dl_append.argtypes = [_vp, ctypes.c_int32, ctypes.POINTER(dl_step_args), _vp]
_lib.dl_eager_step.argtypes = [_vp, ctypes.c_int32, ctypes.POINTER(dl_step_args), _vp]
_lib.dl_merge.argtypes = [_vp, ctypes.c_int32, _vp, ctypes.c_int32, _vp]
_lib.dl_materialize.argtypes = [_vp, ctypes.c_int32, _vp, ctypes.c_int32, _vp, _vp]
_lib.dl_reset_slots.argtypes = [_vp, _vp, ctypes.c_int32, _vp]
_lib.dl_read_error.argtypes = [_vp, ctypes.POINTER(ctypes.c_int32), ctypes.c_int32, _vp]
_lib.dl_decode_step_noalloc.argtypes = [ctypes.POINTER(dl_pool_desc), ctypes.c_int32,
                                        ctypes.POINTER(dl_step_args), ctypes.c_int32, _vp]
_lib.dl_debug_stall.argtypes = [ctypes.c_int64]
_lib.dl_merge_policy.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]
_lib.dl_status_string.argtypes = [ctypes.c_int]
_lib.dl_status_string.restype = ctypes.c_char_p
for _f in ("dl_log_bytes", "dl_create_pool", "dl_destroy_pool", "dl_decode_step", "dl_append", "dl_eager_step",
           "dl_merge", "dl_materialize", "dl_reset_slots", "dl_read_error", "dl_decode_step_noalloc",
           "dl_debug_stall", "dl_merge_policy"):
    getattr(_lib, _f).restype = ctypes.c_int


class DeltaLogError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {dl_status_string(status)} ({status})")


def dl_status_string(status: int) -> str:
    return _lib.dl_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != DL_OK:
        raise DeltaLogError(status, what)


def header_functions() -> list[str]:
    """Names of the functions include/deltalog.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(dl_\w+)\s*\(", text, re.M)))


def library():
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev_tensor(t, name, dtype=None, device=None):
    """A contiguous CUDA tensor of the given dtype, on the pool's device when one is
    given (the library sees only the pointer, so a tensor of another GPU would be
    read through the wrong context)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the pool on {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


class Pool:
    """State pool + log ring + metadata in caller-owned (torch) device memory."""

    def __init__(self, n_slots, n_layers, n_heads, d_k, d_v, log_cap, decay="none",
                 update="add", n_kheads=None, device="cuda", with_log=True, tile_v=0,
                 log_format="fp32", replay="per_tile"):
        dev = torch.device(device)
        n_kheads = n_heads if n_kheads is None else n_kheads
        self.n_slots, self.n_layers, self.n_heads, self.n_kheads = n_slots, n_layers, n_heads, n_kheads
        self.d_k, self.d_v, self.log_cap, self.decay, self.update = d_k, d_v, log_cap, decay, update
        self.tile_v, self.log_format, self.replay = tile_v, log_format, replay
        self.desc = dl_pool_desc(n_slots, n_layers, n_heads, n_kheads, d_k, d_v, log_cap,
                                 DECAY[decay], UPDATE[update], tile_v, LOG_FORMAT[log_format],
                                 REPLAY[replay])
        nbytes = ctypes.c_int64()
        _check(_lib.dl_log_bytes(ctypes.byref(self.desc), ctypes.byref(nbytes)), "dl_log_bytes")
        # one entry in 4-byte words (its bf16 parts, if any, are packed in pairs)
        self.entry_floats = nbytes.value // (4 * n_slots * n_layers * n_heads * log_cap)
        self.state = torch.zeros(n_slots, n_layers, n_heads, d_k, d_v, dtype=torch.float32, device=dev)
        self.log = (torch.zeros(n_slots, n_layers, n_heads, log_cap, self.entry_floats,
                                dtype=torch.float32, device=dev) if with_log else None)
        self.log_len = torch.zeros(n_slots, n_layers, dtype=torch.int32, device=dev)
        self.arrive = torch.zeros(n_slots, n_layers, dtype=torch.int32, device=dev)
        self.err_word = torch.zeros(1, dtype=torch.int32, device=dev)
        self.desc.state = self.state.data_ptr()
        self.desc.log = None if self.log is None else self.log.data_ptr()
        self.desc.log_len = self.log_len.data_ptr()
        self.desc.arrive = self.arrive.data_ptr()
        self.desc.err_word = self.err_word.data_ptr()
        h = ctypes.c_void_p()
        _check(_lib.dl_create_pool(ctypes.byref(self.desc), ctypes.byref(h)), "dl_create_pool")
        self.handle = h

    def close(self):
        if self.handle:
            _check(_lib.dl_destroy_pool(self.handle), "dl_destroy_pool")
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _step_args(pool, slots, q, k, v, lam, beta, out, lambda_per_head):
    dev = pool.state.device
    slots = _dev_tensor(slots, "slots", torch.int32, dev)
    q = _dev_tensor(q, "q", None, dev)
    k = _dev_tensor(k, "k", q.dtype, dev)
    v = _dev_tensor(v, "v", q.dtype, dev)
    if q.dtype not in DTYPE:
        raise TypeError("q/k/v must be float32 or bfloat16")
    lam = _dev_tensor(lam, "lambda", torch.float32, dev)
    beta = _dev_tensor(beta, "beta", torch.float32, dev)
    out = _dev_tensor(out, "out", torch.float32, dev)
    B = slots.numel()
    if q.shape != (B, pool.n_kheads, pool.d_k) or k.shape != q.shape:
        raise ValueError(f"q/k must be [{B}, {pool.n_kheads}, {pool.d_k}]")
    if v.shape != (B, pool.n_heads, pool.d_v):
        raise ValueError(f"v must be [{B}, {pool.n_heads}, {pool.d_v}]")
    if pool.decay != "none":
        lead = (pool.n_heads,) if lambda_per_head else (B, pool.n_heads)
        want = lead if pool.decay == "scalar" else lead + (pool.d_k,)
        if lam is None or tuple(lam.shape) != want:
            raise ValueError(f"lambda must be {list(want)}")
    if pool.update != "add" and (beta is None or tuple(beta.shape) != (B, pool.n_heads)):
        raise ValueError(f"beta must be [{B}, {pool.n_heads}]")
    if out is not None and tuple(out.shape) != (B, pool.n_heads, pool.d_v):
        raise ValueError(f"out must be [{B}, {pool.n_heads}, {pool.d_v}]")
    return dl_step_args(_ptr(slots), B, _ptr(q), _ptr(k), _ptr(v), DTYPE[q.dtype], _ptr(lam),
                        1 if lambda_per_head else 0, _ptr(beta), _ptr(out))


def dl_decode_step(pool: Pool, layer: int, slots, q, k, v, lam=None, beta=None, out=None,
                   lambda_per_head=False, auto_merge=True, stream=None):
    """One decode step of one layer; returns out [B, H, d_v] fp32."""
    if out is None:
        out = torch.empty(slots.numel(), pool.n_heads, pool.d_v, dtype=torch.float32,
                          device=pool.state.device)
    a = _step_args(pool, slots, q, k, v, lam, beta, out, lambda_per_head)
    _check(_lib.dl_decode_step(pool.handle, layer, ctypes.byref(a), merge_code(auto_merge),
                               _stream(stream)), "dl_decode_step")
    return out


def dl_decode_step_noalloc(pool: Pool, layer: int, slots, q, k, v, lam=None, beta=None, out=None,
                           lambda_per_head=False, auto_merge=True, stream=None):
    """dl_decode_step without the caller's arrival-counter buffer: the library keeps
    the counters in a fixed device array of its own (for callers that cannot
    allocate device memory).  The pool's descriptor is passed with `arrive` unset;
    the pool's own `arrive` tensor is not touched.  Calls must not overlap on the
    GPU (they share the array)."""
    if out is None:
        out = torch.empty(slots.numel(), pool.n_heads, pool.d_v, dtype=torch.float32,
                          device=pool.state.device)
    a = _step_args(pool, slots, q, k, v, lam, beta, out, lambda_per_head)
    desc = dl_pool_desc.from_buffer_copy(pool.desc)
    desc.arrive = None
    _check(_lib.dl_decode_step_noalloc(ctypes.byref(desc), layer, ctypes.byref(a),
                                       merge_code(auto_merge), _stream(stream)),
           "dl_decode_step_noalloc")
    return out


def dl_append(pool: Pool, layer: int, slots, q, k, v, lam=None, beta=None,
              lambda_per_head=False, stream=None):
    a = _step_args(pool, slots, q, k, v, lam, beta, None, lambda_per_head)
    _check(_lib.dl_append(pool.handle, layer, ctypes.byref(a), _stream(stream)), "dl_append")


def dl_eager_step(pool: Pool, layer: int, slots, q, k, v, lam=None, beta=None, out=None,
                  lambda_per_head=False, stream=None):
    if out is None:
        out = torch.empty(slots.numel(), pool.n_heads, pool.d_v, dtype=torch.float32,
                          device=pool.state.device)
    a = _step_args(pool, slots, q, k, v, lam, beta, out, lambda_per_head)
    _check(_lib.dl_eager_step(pool.handle, layer, ctypes.byref(a), _stream(stream)),
           "dl_eager_step")
    return out


def dl_merge(pool: Pool, layer: int, slots, stream=None):
    slots = _dev_tensor(slots, "slots", torch.int32, pool.state.device)
    _check(_lib.dl_merge(pool.handle, layer, _ptr(slots), slots.numel(), _stream(stream)),
           "dl_merge")


def dl_materialize(pool: Pool, layer: int, slots, dense_out=None, stream=None):
    dev = pool.state.device
    slots = _dev_tensor(slots, "slots", torch.int32, dev)
    want = (slots.numel(), pool.n_heads, pool.d_k, pool.d_v)
    if dense_out is None:
        dense_out = torch.empty(want, dtype=torch.float32, device=dev)
    dense_out = _dev_tensor(dense_out, "dense_out", torch.float32, dev)
    if tuple(dense_out.shape) != want:
        raise ValueError(f"dense_out must be {list(want)}, got {list(dense_out.shape)}")
    _check(_lib.dl_materialize(pool.handle, layer, _ptr(slots), slots.numel(), _ptr(dense_out),
                               _stream(stream)), "dl_materialize")
    return dense_out


def dl_reset_slots(pool: Pool, slots, stream=None):
    slots = _dev_tensor(slots, "slots", torch.int32, pool.state.device)
    _check(_lib.dl_reset_slots(pool.handle, _ptr(slots), slots.numel(), _stream(stream)),
           "dl_reset_slots")


def dl_read_error(pool: Pool, clear=True, stream=None) -> int:
    """Device error bits (0 when clean); synchronises the stream."""
    bits = ctypes.c_int32(0)
    st = _lib.dl_read_error(pool.handle, ctypes.byref(bits), 1 if clear else 0, _stream(stream))
    if st not in (DL_OK, DL_ERR_DEVICE):
        raise DeltaLogError(st, "dl_read_error")
    return int(bits.value)


def dl_merge_policy(batch: int, n_heads: int, auto_merge="adaptive") -> bool:
    """Whether dl_decode_step of this batch merges every slot on every step."""
    out = ctypes.c_int32(0)
    _check(_lib.dl_merge_policy(int(batch), int(n_heads), merge_code(auto_merge), ctypes.byref(out)),
           "dl_merge_policy")
    return bool(out.value)


def dl_debug_stall(limit_ns: int = 0):
    """Test hook: while limit_ns > 0, each whole-head decode launch makes one warp wait
    (bounded by limit_ns) on a barrier nothing completes, so it takes the kernel's
    timeout path; limit_ns <= 0 switches it off (process-wide)."""
    _check(_lib.dl_debug_stall(int(limit_ns)), "dl_debug_stall")


class PreparedStep:
    """A decode / append / eager call with its argument block built once.

    Calling it issues the C call directly (no per-call marshalling), which keeps host
    overhead out of tight loops such as CUDA-graph capture or back-to-back timing.
    The tensors passed in are kept alive by this object.
    """

    def __init__(self, kind: str, pool: Pool, layer: int, slots, q, k, v, lam=None, beta=None,
                 out=None, lambda_per_head=False, auto_merge=True):
        if kind not in ("decode", "append", "eager"):
            raise ValueError(kind)
        if kind != "append" and out is None:
            out = torch.empty(slots.numel(), pool.n_heads, pool.d_v, dtype=torch.float32,
                              device=pool.state.device)
        self._keep = (slots, q, k, v, lam, beta, out)
        self.out = out
        self.pool, self.layer, self.kind = pool, int(layer), kind
        self.args = _step_args(pool, slots, q, k, v, lam, beta, None if kind == "append" else out,
                               lambda_per_head)
        self._ref = ctypes.byref(self.args)
        self._auto = merge_code(auto_merge)

    def __call__(self, stream=None) -> int:
        st = _stream(stream)
        if self.kind == "decode":
            return _lib.dl_decode_step(self.pool.handle, self.layer, self._ref, self._auto, st)
        if self.kind == "append":
            return _lib.dl_append(self.pool.handle, self.layer, self._ref, st)
        return _lib.dl_eager_step(self.pool.handle, self.layer, self._ref, st)
