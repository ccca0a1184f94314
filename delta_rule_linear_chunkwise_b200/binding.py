"""ctypes binding of libdr.so (the C ABI in ``include/dr.h``).

Argument marshalling only: every step of the operator runs in the library's
CUDA kernels.  PyTorch supplies device memory (inputs, outputs and the scratch
workspace) and the stream.  There is no fallback: if ``libdr.so`` is missing or
a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdr.so")

DR_OK, DR_ERR_INVALID_ARG, DR_ERR_UNSUPPORTED, DR_ERR_WORKSPACE, DR_ERR_CUDA, DR_ERR_TIMEOUT = range(6)
DR_F32, DR_BF16 = 0, 1
GATES = {"none": 0, "scalar": 1, "channel": 2, "phase": 3}
BETA_MODES = {"direct": 0, "kaczmarz": 1}


class DrProblem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("chunk", ctypes.c_int),
                ("dtype", ctypes.c_int), ("gate", ctypes.c_int), ("beta_mode", ctypes.c_int),
                ("eps", ctypes.c_float)]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int),
                ("ms_total", ctypes.c_double), ("bytes_per_launch", ctypes.c_double),
                ("flops_per_launch", ctypes.c_double),
                ("design_bytes_per_launch", ctypes.c_double)]


class DrError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def load() -> ctypes.CDLL:
    """Load libdr.so from the package directory (built by ``build.py``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m delta_rule_linear_chunkwise_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(DrProblem)
    vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    lib.dr_workspace_size.argtypes = [P, i, ctypes.POINTER(sz)]
    lib.dr_workspace_size.restype = i
    lib.dr_saved_size.argtypes = [P, ctypes.POINTER(sz)]
    lib.dr_saved_size.restype = i
    lib.dr_chunk_fwd.argtypes = [P] + [vp] * 9 + [vp, sz, vp]
    lib.dr_chunk_fwd.restype = i
    lib.dr_chunk_bwd.argtypes = [P] + [vp] * 15 + [vp, sz, vp]
    lib.dr_chunk_bwd.restype = i
    lib.dr_decode_step.argtypes = [P] + [vp] * 7 + [vp]
    lib.dr_decode_step.restype = i
    lib.dr_status_string.argtypes = [i]
    lib.dr_status_string.restype = ctypes.c_char_p
    lib.dr_last_device_error.argtypes = [vp]
    lib.dr_last_device_error.restype = i
    lib.dr_inject_timeout.argtypes = [i]
    lib.dr_inject_timeout.restype = i
    lib.dr_version.argtypes = []
    lib.dr_version.restype = i
    lib.dr_profile_enable.argtypes = [i]
    lib.dr_profile_enable.restype = i
    lib.dr_profile_read.argtypes = [ctypes.POINTER(KernelTime), i]
    lib.dr_profile_read.restype = i
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().dr_status_string(status).decode()


def _check(status: int, what: str):
    if status != DR_OK:
        raise DrError(status, what)


def make_problem(B, H, T, dk, dv, *, dtype="bf16", gate="scalar", beta_mode="direct",
                 eps=1e-6, chunk=64) -> DrProblem:
    return DrProblem(B, H, T, dk, dv, chunk, DR_BF16 if dtype == "bf16" else DR_F32,
                     GATES[gate], BETA_MODES[beta_mode], eps)


def workspace_size(prob: DrProblem, pass_: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().dr_workspace_size(ctypes.byref(prob), pass_, ctypes.byref(n)),
           "dr_workspace_size")
    return n.value


def saved_size(prob: DrProblem) -> int:
    n = ctypes.c_size_t(0)
    _check(load().dr_saved_size(ctypes.byref(prob), ctypes.byref(n)), "dr_saved_size")
    return n.value


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype, shape, device):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")


@dataclass
class Plan:
    """A problem description plus reusable workspaces for repeated calls."""
    B: int
    H: int
    T: int
    dk: int
    dv: int
    dtype: str = "bf16"
    gate: str = "scalar"
    beta_mode: str = "direct"
    eps: float = 1e-6
    chunk: int = 64
    device: str | torch.device = "cuda"

    def __post_init__(self):
        self.device = torch.device(self.device)
        if self.device.type == "cuda" and self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        self.prob = make_problem(self.B, self.H, self.T, self.dk, self.dv, dtype=self.dtype,
                                 gate=self.gate, beta_mode=self.beta_mode, eps=self.eps,
                                 chunk=self.chunk)
        self.tdtype = torch.bfloat16 if self.dtype == "bf16" else torch.float32
        self._ws = {}

    @classmethod
    def for_workload(cls, w, device="cuda"):
        return cls(w.B, w.H, w.T, w.dk, w.dv, dtype=w.dtype, gate=w.gate,
                   beta_mode=w.beta_mode, eps=w.eps, chunk=w.chunk, device=device)

    def workspace(self, pass_: int) -> torch.Tensor:
        if pass_ not in self._ws:
            n = workspace_size(self.prob, pass_)
            self._ws[pass_] = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
        return self._ws[pass_]

    def new_saved(self) -> torch.Tensor:
        return torch.empty(saved_size(self.prob), dtype=torch.uint8, device=self.device)

    def _shapes(self):
        B, T, H, dk, dv = self.B, self.T, self.H, self.dk, self.dv
        g = None if self.gate == "none" else \
            ((B, T, H, dk) if self.gate in ("channel", "phase") else (B, T, H))
        return (B, T, H, dk), (B, T, H, dv), (B, T, H), g, (B, H, dv, dk)

    def _check_inputs(self, q, k, v, beta, g, S0):
        sq, sv, sb, sg, ss = self._shapes()
        _need(q, "q", self.tdtype, sq, self.device)
        _need(k, "k", self.tdtype, sq, self.device)
        _need(v, "v", self.tdtype, sv, self.device)
        _need(beta, "beta", torch.float32, sb, self.device)
        if sg is None:
            if g is not None:
                raise ValueError("g must be None for gate 'none'")
        else:
            _need(g, "g", torch.float32, sg, self.device)
        if S0 is not None:
            _need(S0, "S0", torch.float32, ss, self.device)

    def fwd(self, q, k, v, beta, g=None, S0=None, *, o=None, ST=None, saved=None,
            want_state=True, save=True, stream=None):
        """dr_chunk_fwd.  Returns ``(o, S_T or None, saved or None)``."""
        self._check_inputs(q, k, v, beta, g, S0)
        _, sv, _, _, ss = self._shapes()
        if o is None:
            o = torch.empty(sv, dtype=self.tdtype, device=self.device)
        if ST is None and want_state:
            ST = torch.empty(ss, dtype=torch.float32, device=self.device)
        if saved is None and save:
            saved = self.new_saved()
        ws = self.workspace(0)
        _check(load().dr_chunk_fwd(ctypes.byref(self.prob), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(beta), _ptr(g), _ptr(S0), _ptr(o), _ptr(ST),
                                   _ptr(saved), _ptr(ws), ws.numel(), _stream(stream)),
               "dr_chunk_fwd")
        return o, ST, saved

    def bwd(self, q, k, v, beta, g, S0, dO, dST=None, saved=None, *, out=None,
            want_dS0=True, stream=None):
        """dr_chunk_bwd.  Returns a dict ``dq, dk, dv, dbeta, dg, dS0``."""
        self._check_inputs(q, k, v, beta, g, S0)
        sq, sv, sb, sg, ss = self._shapes()
        _need(dO, "dO", self.tdtype, sv, self.device)
        if dST is not None:
            _need(dST, "dST", torch.float32, ss, self.device)
        if out is None:
            out = dict(dq=torch.empty(sq, dtype=self.tdtype, device=self.device),
                       dk=torch.empty(sq, dtype=self.tdtype, device=self.device),
                       dv=torch.empty(sv, dtype=self.tdtype, device=self.device),
                       dbeta=torch.empty(sb, dtype=torch.float32, device=self.device),
                       dg=None if sg is None else torch.empty(sg, dtype=torch.float32,
                                                              device=self.device),
                       dS0=torch.empty(ss, dtype=torch.float32, device=self.device)
                       if want_dS0 else None)
        ws = self.workspace(1)
        _check(load().dr_chunk_bwd(ctypes.byref(self.prob), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(beta), _ptr(g), _ptr(S0), _ptr(dO), _ptr(dST),
                                   _ptr(saved), _ptr(out["dq"]), _ptr(out["dk"]),
                                   _ptr(out["dv"]), _ptr(out["dbeta"]), _ptr(out["dg"]),
                                   _ptr(out["dS0"]), _ptr(ws), ws.numel(), _stream(stream)),
               "dr_chunk_bwd")
        return out


def last_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return load().dr_last_device_error(_stream(stream))


def _gate_of(g, gate):
    if gate is not None:
        return gate
    return "none" if g is None else ("channel" if g.dim() == 4 else "scalar")


def chunk_fwd(q, k, v, beta, g=None, S0=None, *, beta_mode="direct", eps=1e-6, chunk=64,
              save=True, stream=None, gate=None):
    """One-shot forward: ``(o, S_T, saved)`` for inputs laid out as in include/dr.h.
    ``gate="phase"`` reads g as the SFDA rotation-decay gate (same shape as the
    per-channel gate); otherwise the gate kind follows from g's shape."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    gate = _gate_of(g, gate)
    dtype = "bf16" if q.dtype == torch.bfloat16 else "f32"
    plan = Plan(B, H, T, dk, dv, dtype=dtype, gate=gate, beta_mode=beta_mode, eps=eps,
                chunk=chunk, device=q.device)
    return plan.fwd(q, k, v, beta, g, S0, save=save, stream=stream)


def chunk_bwd(q, k, v, beta, g, S0, dO, dST=None, saved=None, *, beta_mode="direct",
              eps=1e-6, chunk=64, stream=None, gate=None):
    """One-shot backward: dict of ``dq, dk, dv, dbeta, dg, dS0``."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    gate = _gate_of(g, gate)
    dtype = "bf16" if q.dtype == torch.bfloat16 else "f32"
    plan = Plan(B, H, T, dk, dv, dtype=dtype, gate=gate, beta_mode=beta_mode, eps=eps,
                chunk=chunk, device=q.device)
    return plan.bwd(q, k, v, beta, g, S0, dO, dST, saved, stream=stream)


def decode_step(q, k, v, beta, g, S, *, beta_mode="direct", eps=1e-6, o=None, stream=None,
                gate=None):
    """One token per head through the recurrent update, S updated in place.

    q, k ``[B,1,H,dk]``, v ``[B,1,H,dv]`` (bf16 or fp32), beta ``[B,1,H]``,
    g ``None`` / ``[B,1,H]`` / ``[B,1,H,dk]`` fp32 (``gate="phase"`` for the
    SFDA rotation-decay gate), S ``[B,H,dv,dk]`` fp32.
    Returns o ``[B,1,H,dv]`` in the storage dtype."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    tdt = q.dtype
    gate = _gate_of(g, gate)
    prob = make_problem(B, H, T, dk, dv, dtype="bf16" if tdt == torch.bfloat16 else "f32",
                        gate=gate, beta_mode=beta_mode, eps=eps)
    _need(q, "q", tdt, (B, 1, H, dk), dev)
    _need(k, "k", tdt, (B, 1, H, dk), dev)
    _need(v, "v", tdt, (B, 1, H, dv), dev)
    _need(beta, "beta", torch.float32, (B, 1, H), dev)
    if g is not None:
        _need(g, "g", torch.float32,
              (B, 1, H, dk) if gate in ("channel", "phase") else (B, 1, H), dev)
    _need(S, "S", torch.float32, (B, H, dv, dk), dev)
    if o is None:
        o = torch.empty(B, 1, H, dv, dtype=tdt, device=dev)
    else:
        _need(o, "o", tdt, (B, 1, H, dv), dev)
    _check(load().dr_decode_step(ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                 _ptr(g), _ptr(S), _ptr(o), _stream(stream)), "dr_decode_step")
    return o


def inject_timeout(launches: int = 1) -> None:
    """Make the next ``launches`` chunk-backward launches take their bounded-wait
    timeout path (fault injection for tests; see ``dr_inject_timeout``)."""
    _check(load().dr_inject_timeout(launches), "dr_inject_timeout")


def profile_enable(on: bool = True) -> None:
    """Bracket every library launch with CUDA events on its stream (or stop)."""
    _check(load().dr_profile_enable(1 if on else 0), "dr_profile_enable")


def profile_read() -> list[dict]:
    """Per-kernel launches, summed event time and work model since the last read:
    ``bytes_per_launch`` is the operator's own inputs and outputs the launch
    touches (algorithmic), ``design_bytes_per_launch`` all it moves by design."""
    buf = (KernelTime * 64)()
    n = load().dr_profile_read(buf, 64)
    if n < 0:
        raise DrError(DR_ERR_CUDA, "dr_profile_read")
    return [dict(name=buf[i].name.decode(), launches=buf[i].launches,
                 ms_total=buf[i].ms_total, bytes_per_launch=buf[i].bytes_per_launch,
                 flops_per_launch=buf[i].flops_per_launch,
                 design_bytes_per_launch=buf[i].design_bytes_per_launch) for i in range(n)]
