"""ctypes wrapper around the float64 C oracle ``kda_ref.c``.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The recurrence it evaluates, per sequence and head, token by token
(Kimi Linear summary, §3 "Kimi Delta Attention"; Kimi K3 architecture
summary, lower-bounded gate; Kimi Linear summary, §4 for the unit-length
normalisation of q and k):

    k^ = k / sqrt(|k|^2 + 1e-6),  q^ likewise
    g  = -5 * sigmoid(exp(A_h) * z),  alpha = exp(g)
    S' = Diag(alpha) S
    S  = (I - beta k^ k^T) S' + beta k^ v^T
    o  = S^T q^

Inputs are numpy arrays; they are widened to float64 here (exact for fp32 and
bf16 values).  ``build()`` compiles the C file with gcc into ``oracle/_build``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_ref.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libkda_ref.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile kda_ref.c into oracle/_build/libkda_ref.so (gcc, -O3)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O3", "-march=native", "-fno-fast-math", "-std=c99",
           "-D_GNU_SOURCE", "-shared", "-fPIC", "-pthread", "-o", tmp, _SRC,
           "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.kda_ref_forward.argtypes = [dp, dp, dp, dp, dp, dp, dp, ip, i64, i64,
                                        i64, i64, i64, dp, dp, dp, ctypes.c_int]
        lib.kda_ref_forward.restype = ctypes.c_int
        lib.kda_ref_forward_g.argtypes = [dp, dp, dp, dp, dp, dp, ip, i64, i64,
                                          i64, i64, i64, dp, dp, dp, ctypes.c_int]
        lib.kda_ref_forward_g.restype = ctypes.c_int
        lib.kda_ref_gate.argtypes = [dp, dp, i64, i64, i64, dp]
        lib.kda_ref_gate.restype = None
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (any dtype) -> exact float64
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, ty=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ty))


def _threads(threads):
    if threads is None or threads <= 0:
        return os.cpu_count() or 1
    return int(threads)


def _cu(cu_seqlens, N, T):
    if cu_seqlens is None:
        if N <= 0 or T % N:
            raise ValueError("equal-length batch needs T divisible by N")
        L = T // N
        return np.arange(0, T + 1, L, dtype=np.int64) if L else np.zeros(N + 1, np.int64)
    cu = np.ascontiguousarray(np.asarray(
        cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
        dtype=np.int64))
    if cu.shape != (N + 1,):
        raise ValueError("cu_seqlens must have N+1 entries")
    return cu


def gate(z, A):
    """g = -5 * sigmoid(exp(A_h) * z) for z [T,H,dk], A [H] (float64)."""
    z = _f64(z)
    A = _f64(A)
    T, H, dk = z.shape
    g = np.empty_like(z)
    _load().kda_ref_gate(_ptr(z), _ptr(A), T, H, dk, _ptr(g))
    return g


def forward(q, k, v, beta, *, z=None, A=None, g=None, S0=None, cu_seqlens=None,
            num_seqs=None, trace=False, threads=None):
    """Sequential float64 KDA over packed sequences.

    q, k, (z or g): [T,H,dk]; v: [T,H,dv]; beta: [T,H]; A: [H];
    S0: [N,H,dk,dv] or None (zeros); cu_seqlens: [N+1] or None (N equal
    sequences, ``num_seqs`` required).  Returns (o [T,H,dv], S_final
    [N,H,dk,dv]) and, when ``trace``, also S after every token [T,H,dk,dv].
    """
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        N = int(num_seqs if num_seqs is not None else (S0.shape[0] if S0 is not None else 1))
    else:
        N = len(cu_seqlens) - 1
    cu = _cu(cu_seqlens, N, T)
    S0 = _f64(S0)
    if S0 is not None and S0.shape != (N, H, dk, dv):
        raise ValueError(f"S0 shape {S0.shape} != {(N, H, dk, dv)}")
    o = np.zeros((T, H, dv), np.float64)
    Sf = np.zeros((N, H, dk, dv), np.float64)
    St = np.zeros((T, H, dk, dv), np.float64) if trace else None
    lib = _load()
    if g is not None:
        g = _f64(g)
        rc = lib.kda_ref_forward_g(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                   _ptr(S0), _ptr(cu, ctypes.c_int64), N, T, H,
                                   dk, dv, _ptr(o), _ptr(Sf), _ptr(St),
                                   _threads(threads))
    else:
        z, A = _f64(z), _f64(A)
        rc = lib.kda_ref_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A),
                                 _ptr(beta), _ptr(S0), _ptr(cu, ctypes.c_int64),
                                 N, T, H, dk, dv, _ptr(o), _ptr(Sf), _ptr(St),
                                 _threads(threads))
    if rc != 0:
        raise ValueError("kda_ref: invalid arguments")
    return (o, Sf, St) if trace else (o, Sf)


def decode_step(q, k, v, beta, S, *, z=None, A=None, g=None, threads=None):
    """One recurrent token per sequence: q,k,z [B,H,dk], v [B,H,dv], beta [B,H],
    S [B,H,dk,dv] (float64, not modified).  Returns (o [B,H,dv], S_new)."""
    q = _f64(q)
    B = q.shape[0]
    cu = np.arange(B + 1, dtype=np.int64)
    return forward(q, k, v, beta, z=z, A=A, g=g, S0=S, cu_seqlens=cu,
                   threads=threads)
