"""fp64 CPU oracle for chunkwise gated delta-rule linear attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never loads it, and it loads nothing from the CUDA library: the two share no
code, headers, tables or helpers.

Two independent restatements live here:

* ``recurrent_fwd`` / ``recurrent_bwd`` -- the plain token-by-token definition
  of the recurrence and a hand-derived reverse-mode pass of it, in C
  (``dr_oracle.c``, fp64, OpenMP over batch x head).  This is *the* oracle the
  CUDA path is compared against.
* ``chunkwise.py`` -- an fp64 numpy restatement of the chunkwise WY/UT form
  and of the triangular-residual backward.  It exists only so the tests can pin
  "chunkwise equals recurrent in exact arithmetic" (ReWY abstract, paperdot
  listing; "Exakter Affiner Chunk-Transfer" and "Ergebnisse" sections of the SFDA
  explainer, gist.science), never as a comparison target for the GPU.

Layouts: q, k ``[B, T, H, dk]``; v, o, dO ``[B, T, H, dv]``; beta ``[B, T, H]``;
g ``[B, T, H]`` (scalar gate) or ``[B, T, H, dk]`` (per-channel gate; also the
phase gate of SFDA, selected with ``gate=GATE_PHASE``: log alpha_j at channel
2j and the phase theta_j at 2j+1 of key pair j) or ``None`` (no gate); states
``[B, H, dv, dk]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

GATE_NONE, GATE_SCALAR, GATE_CHANNEL, GATE_PHASE = 0, 1, 2, 3
BETA_DIRECT, BETA_KACZMARZ = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dr_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``dr_oracle.c`` into ``liboracle.so`` next to it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.oracle_fwd.argtypes = [i, i, i, i, i, i, i, ctypes.c_double] + [dp] * 8
        lib.oracle_fwd.restype = i
        lib.oracle_bwd.argtypes = [i, i, i, i, i, i, i, ctypes.c_double] + [dp] * 14
        lib.oracle_bwd.restype = i
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    if x is None:
        return ctypes.POINTER(ctypes.c_double)()
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def gate_kind(g, dk: int, gate=None) -> int:
    """The gate kind: ``gate`` when given (needed for the phase gate, which has
    the per-channel gate's shape), else inferred from the shape of ``g``."""
    if g is None:
        return GATE_NONE
    if gate is not None:
        if gate == GATE_PHASE and (g.ndim != 4 or g.shape[-1] != dk or dk % 2):
            raise ValueError("phase gate: g must be [B, T, H, dk] with dk even")
        return gate
    return GATE_CHANNEL if (g.ndim == 4 and g.shape[-1] == dk) else GATE_SCALAR


def _dims(q, v):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    return B, T, H, dk, dv


def recurrent_fwd(q, k, v, beta, g=None, S0=None, beta_mode=BETA_DIRECT, eps=1e-6,
                  return_threads=False, gate=None):
    """Token-by-token forward.  Returns ``(o, S_T)`` as fp64 arrays.

    ``gate=GATE_PHASE`` selects the SFDA rotation-decay gate: ``g[..., 2j]`` is
    log alpha_j and ``g[..., 2j+1]`` the phase theta_j of key pair j."""
    q, k, v, beta, g, S0 = map(_f64, (q, k, v, beta, g, S0))
    B, T, H, dk, dv = _dims(q, v)
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    used = _load().oracle_fwd(B, H, T, dk, dv, gate_kind(g, dk, gate), beta_mode, eps,
                              _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S0),
                              _ptr(o), _ptr(ST))
    return (o, ST, used) if return_threads else (o, ST)


def recurrent_bwd(q, k, v, beta, g, S0, dO, dST=None, beta_mode=BETA_DIRECT, eps=1e-6,
                  return_threads=False, gate=None):
    """Hand-derived reverse mode of the recurrence.

    Returns a dict with ``dq, dk, dv, dbeta, dg, dS0`` (``dg`` is ``None`` when
    there is no gate; in Kaczmarz mode ``dbeta`` is the gradient w.r.t. eta;
    for the phase gate ``dg[..., 2j]`` is d/d log alpha_j and ``dg[..., 2j+1]``
    d/d theta_j).
    """
    q, k, v, beta, g, S0, dO, dST = map(_f64, (q, k, v, beta, g, S0, dO, dST))
    B, T, H, dk, dv = _dims(q, v)
    gk = gate_kind(g, dk, gate)
    dq = np.zeros_like(q)
    dkk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    db = np.zeros((B, T, H))
    dg = None if g is None else np.zeros_like(g)
    dS0 = np.zeros((B, H, dv, dk))
    used = _load().oracle_bwd(B, H, T, dk, dv, gk, beta_mode, eps,
                              _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(S0),
                              _ptr(dO), _ptr(dST), _ptr(dq), _ptr(dkk), _ptr(dvv),
                              _ptr(db), _ptr(dg), _ptr(dS0))
    out = dict(dq=dq, dk=dkk, dv=dvv, dbeta=db, dg=dg, dS0=dS0)
    if return_threads:
        out["threads"] = used
    return out
