"""CPU oracle for the recurrent-state decode step (fp64).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline / reference legs use it; the product path never imports it.

* ``eager_rollout`` -- the plain definition: the eager recurrence of the common
  decode form (DeltaLog paper, "Background"), written in C (``eager.c``) and run
  over many independent (slot, layer, head) trajectories with OpenMP.
* ``deferred`` -- an independent fp64 implementation of the append-merge cycle
  (DeltaLog paper, "Append-merge decoding" and the logical-state equation of
  its traffic model), used only to pin the eager oracle and the log layout.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "eager.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DECAY = {"none": 0, "scalar": 1, "diag": 2}
UPDATE = {"add": 0, "delta": 1, "delta_undecayed": 2}


class _Dims(ctypes.Structure):
    _fields_ = [("d_k", ctypes.c_int), ("d_v", ctypes.c_int), ("steps", ctypes.c_int),
                ("decay", ctypes.c_int), ("update", ctypes.c_int), ("n_ckpt", ctypes.c_int)]


def compile_c(src: str = _SRC, out: str = _LIB, extra=()) -> str:
    """gcc -O2 -fopenmp; fp64 throughout, no fast-math."""
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", *extra, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


_lib = None


def load(path: str | None = None):
    """Load (building if missing or stale) the C oracle."""
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
    else:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            compile_c()
        lib = ctypes.CDLL(_LIB)
    lib.oracle_eager_run.restype = ctypes.c_int
    lib.oracle_eager_run.argtypes = [ctypes.POINTER(_Dims), ctypes.c_long] + \
        [ctypes.c_void_p] * 7 + [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.oracle_max_threads.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def max_threads() -> int:
    return load().oracle_max_threads()


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def eager_tasks(S0, q, k, v, lam, beta, *, decay: str, update: str, ckpts=(),
                threads: int = 0, lib=None):
    """Run n independent trajectories.

    S0 [n, d_k, d_v]; q, k [n, T, d_k]; v [n, T, d_v]; lam None | [n, T] (scalar)
    | [n, T, d_k] (diag); beta None | [n, T].  All float64.
    Returns (out [n, T, d_v], S_ckpt [n, len(ckpts), d_k, d_v]).
    """
    lib = lib or load()
    S0 = np.ascontiguousarray(S0, np.float64)
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    n, dk, dv = S0.shape
    T = q.shape[1]
    assert q.shape == (n, T, dk) and k.shape == (n, T, dk) and v.shape == (n, T, dv)
    if decay != "none":
        lam = np.ascontiguousarray(lam, np.float64)
        assert lam.shape == ((n, T) if decay == "scalar" else (n, T, dk)), lam.shape
    else:
        lam = None
    if update != "add":
        beta = np.ascontiguousarray(beta, np.float64)
        assert beta.shape == (n, T)
    else:
        beta = None
    ck = np.ascontiguousarray(np.asarray(ckpts, dtype=np.int32).reshape(-1))
    out = np.zeros((n, T, dv), np.float64)
    S_ck = np.zeros((n, len(ck), dk, dv), np.float64)
    dims = _Dims(dk, dv, T, DECAY[decay], UPDATE[update], len(ck))
    rc = lib.oracle_eager_run(ctypes.byref(dims), n, _ptr(S0), _ptr(q), _ptr(k), _ptr(v),
                              _ptr(lam), _ptr(beta), _ptr(ck) if len(ck) else None,
                              _ptr(out), _ptr(S_ck) if len(ck) else None, int(threads))
    if rc != 0:
        raise RuntimeError("oracle_eager_run failed")
    return out, S_ck


def eager_rollout(S0, Q, K, V, LAM, BETA, *, decay: str, update: str,
                  lambda_const: bool = False, ckpts=(), threads: int = 0, lib=None):
    """Batched form over the serving layout of one layer.

    S0 [B, H, d_k, d_v]; Q, K [T, B, H_k, d_k]; V [T, B, H, d_v];
    LAM None | [T, B, H] (scalar) | [T, B, H, d_k] (diag) | [H] / [H, d_k] when
    lambda_const (one log-decay per head for all steps and slots);
    BETA None | [T, B, H].  All float64.

    Grouped value attention: v-head h reads q/k of k-head h // (H / H_k)
    (FPGA paper, Fig. 3: paired v-heads share one q/k datapath).

    Returns (O [T, B, H, d_v], S_ckpt [len(ckpts), B, H, d_k, d_v]).
    """
    B, H, dk, dv = S0.shape
    T, _, Hk, _ = Q.shape
    if H % Hk:
        raise ValueError("n_heads must be a multiple of n_kheads")
    kh = np.arange(H) // (H // Hk)
    q = np.transpose(Q[:, :, kh, :], (1, 2, 0, 3)).reshape(B * H, T, dk)
    k = np.transpose(K[:, :, kh, :], (1, 2, 0, 3)).reshape(B * H, T, dk)
    v = np.transpose(V, (1, 2, 0, 3)).reshape(B * H, T, dv)
    lam = None
    if decay != "none":
        L = np.asarray(LAM, np.float64)
        if lambda_const:
            L = np.broadcast_to(L, (T, B) + L.shape)
        if decay == "scalar":
            lam = np.transpose(L, (1, 2, 0)).reshape(B * H, T)
        else:
            lam = np.transpose(L, (1, 2, 0, 3)).reshape(B * H, T, dk)
    beta = None
    if update != "add":
        beta = np.transpose(np.asarray(BETA, np.float64), (1, 2, 0)).reshape(B * H, T)
    out, S_ck = eager_tasks(S0.reshape(B * H, dk, dv), q, k, v, lam, beta, decay=decay,
                            update=update, ckpts=ckpts, threads=threads, lib=lib)
    O = np.transpose(out.reshape(B, H, T, dv), (2, 0, 1, 3))
    S = np.transpose(S_ck.reshape(B, H, len(ckpts), dk, dv), (2, 0, 1, 3, 4))
    return O, S
