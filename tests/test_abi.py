"""The C ABI (include/dr.h): the library loads without a GPU, exports every
declared entry point, sizes its buffers, and rejects bad arguments on the host
before launching anything.  No call here reaches a kernel."""
import ctypes
import os
import re

import pytest

from delta_rule_linear_chunkwise_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(dr_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"dr_chunk_fwd", "dr_chunk_bwd", "dr_workspace_size", "dr_saved_size",
            "dr_status_string", "dr_last_device_error", "dr_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.dr_version() >= 100
    for s in range(6):
        assert len(binding.status_string(s)) > 0
    assert binding.status_string(99) == "unknown status"


def _prob(**kw):
    base = dict(B=2, H=3, T=130, dk=64, dv=32, dtype="bf16", gate="channel",
                beta_mode="direct", eps=1e-6, chunk=64)
    base.update(kw)
    return binding.make_problem(base.pop("B"), base.pop("H"), base.pop("T"), base.pop("dk"),
                                base.pop("dv"), **base)


def test_workspace_sizes_scale_with_problem(lib):
    p = _prob()
    f, b, s = binding.workspace_size(p, 0), binding.workspace_size(p, 1), binding.saved_size(p)
    assert 0 < f < b and s > 0 and f % 256 == 0 and b % 256 == 0
    # saved states: B*H*ceil(T/64) chunk states of dv x dk fp32
    assert s >= 2 * 3 * 3 * 32 * 64 * 4
    p2 = _prob(T=260)
    assert binding.workspace_size(p2, 1) > b


@pytest.mark.parametrize("kw,status", [
    (dict(chunk=32), binding.DR_ERR_UNSUPPORTED),
    (dict(dk=100), binding.DR_ERR_UNSUPPORTED),
    (dict(dv=256), binding.DR_ERR_UNSUPPORTED),
    (dict(T=0), binding.DR_ERR_INVALID_ARG),
    (dict(B=-1), binding.DR_ERR_INVALID_ARG),
    (dict(eps=-1.0), binding.DR_ERR_INVALID_ARG),
])
def test_bad_problems_rejected(lib, kw, status):
    p = _prob(**kw)
    n = ctypes.c_size_t(0)
    assert lib.dr_workspace_size(ctypes.byref(p), 0, ctypes.byref(n)) == status
    assert lib.dr_saved_size(ctypes.byref(p), ctypes.byref(n)) == status


def test_bad_pass_and_null_problem(lib):
    n = ctypes.c_size_t(0)
    assert lib.dr_workspace_size(ctypes.byref(_prob()), 2, ctypes.byref(n)) == binding.DR_ERR_INVALID_ARG
    assert lib.dr_workspace_size(None, 0, ctypes.byref(n)) == binding.DR_ERR_INVALID_ARG
    assert lib.dr_workspace_size(ctypes.byref(_prob()), 0, None) == binding.DR_ERR_INVALID_ARG


# Fake, never-dereferenced device addresses: validation happens on the host
# before any launch, so these calls fail with a status and touch no memory.
A = 0x7F0000000000


def _fwd(lib, p, **over):
    args = dict(q=A, k=A + 0x1000, v=A + 0x2000, beta=A + 0x3000, g=A + 0x4000, S0=None,
                o=A + 0x5000, ST=None, saved=None, ws=A + 0x10000, ws_bytes=1 << 40)
    args.update(over)
    vp = ctypes.c_void_p
    return lib.dr_chunk_fwd(ctypes.byref(p), *(vp(args[n]) if args[n] else None for n in
                            ("q", "k", "v", "beta", "g", "S0", "o", "ST", "saved", "ws")),
                            args["ws_bytes"], None)


def _bwd(lib, p, **over):
    names = ("q", "k", "v", "beta", "g", "S0", "dO", "dST", "saved", "dq", "dk", "dv",
             "dbeta", "dg", "dS0", "ws")
    args = {n: A + 0x1000 * i for i, n in enumerate(names)}
    args.update(S0=None, dST=None, saved=None, dS0=None, ws=A + 0x100000, ws_bytes=1 << 40)
    args.update(over)
    vp = ctypes.c_void_p
    return lib.dr_chunk_bwd(ctypes.byref(p), *(vp(args[n]) if args[n] else None for n in names),
                            args["ws_bytes"], None)


def test_fwd_argument_errors(lib):
    p = _prob()
    assert _fwd(lib, p, q=None) == binding.DR_ERR_INVALID_ARG
    assert _fwd(lib, p, o=None) == binding.DR_ERR_INVALID_ARG
    assert _fwd(lib, p, g=None) == binding.DR_ERR_INVALID_ARG          # gate needs g
    assert _fwd(lib, _prob(gate="none")) == binding.DR_ERR_INVALID_ARG  # no gate, g given
    assert _fwd(lib, p, k=A + 8) == binding.DR_ERR_INVALID_ARG          # misaligned
    assert _fwd(lib, p, ws=None) == binding.DR_ERR_WORKSPACE
    assert _fwd(lib, p, ws_bytes=binding.workspace_size(p, 0) - 1) == binding.DR_ERR_WORKSPACE
    assert _fwd(lib, p, ws=A + 0x10010) == binding.DR_ERR_WORKSPACE    # not 256-aligned
    assert _fwd(lib, _prob(chunk=16)) == binding.DR_ERR_UNSUPPORTED


def test_bwd_argument_errors(lib):
    p = _prob()
    assert _bwd(lib, p, dO=None) == binding.DR_ERR_INVALID_ARG
    assert _bwd(lib, p, dbeta=None) == binding.DR_ERR_INVALID_ARG
    assert _bwd(lib, p, dg=None) == binding.DR_ERR_INVALID_ARG          # gated needs dg
    assert _bwd(lib, p, dq=A + 4) == binding.DR_ERR_INVALID_ARG
    assert _bwd(lib, p, ws_bytes=binding.workspace_size(p, 1) - 256) == binding.DR_ERR_WORKSPACE
    assert _bwd(lib, _prob(dk=48, dv=24)) == binding.DR_ERR_UNSUPPORTED


def _dec(lib, p, **over):
    names = ("q", "k", "v", "beta", "g", "S", "o")
    args = {n: A + 0x1000 * i for i, n in enumerate(names)}
    args.update(over)
    vp = ctypes.c_void_p
    return lib.dr_decode_step(ctypes.byref(p), *(vp(args[n]) if args[n] else None for n in names),
                              None)


def test_decode_argument_errors(lib):
    p = _prob(T=1)
    assert _dec(lib, _prob(T=2)) == binding.DR_ERR_INVALID_ARG         # one token per call
    assert _dec(lib, p, S=None) == binding.DR_ERR_INVALID_ARG          # the state is in/out
    assert _dec(lib, p, o=None) == binding.DR_ERR_INVALID_ARG
    assert _dec(lib, p, g=None) == binding.DR_ERR_INVALID_ARG          # gate needs g
    assert _dec(lib, _prob(T=1, gate="none")) == binding.DR_ERR_INVALID_ARG  # no gate, g given
    assert _dec(lib, p, v=A + 0x2004) == binding.DR_ERR_INVALID_ARG    # misaligned
    assert _dec(lib, _prob(T=1, dk=24)) == binding.DR_ERR_UNSUPPORTED


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "libdr.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        binding.load()


def test_phase_gate_routing(lib):
    # The SFDA phase gate: forward and backward on the bf16 d = 128 tensor-core
    # path only; an unknown gate value is an argument error.  Host-side checks
    # only (fake pointers: every call here must be rejected before a launch).
    assert _fwd(lib, _prob(gate="phase")) == binding.DR_ERR_UNSUPPORTED          # dk = 64
    assert _fwd(lib, _prob(gate="phase", dk=128, dv=128, dtype="f32")) == \
        binding.DR_ERR_UNSUPPORTED
    assert _bwd(lib, _prob(gate="phase")) == binding.DR_ERR_UNSUPPORTED          # dk = 64
    assert _bwd(lib, _prob(gate="phase", dk=128, dv=128, dtype="f32")) == \
        binding.DR_ERR_UNSUPPORTED
    assert _bwd(lib, _prob(gate="phase", dk=128, dv=128), dg=None) == binding.DR_ERR_INVALID_ARG
    assert _fwd(lib, _prob(gate="phase", dk=128, dv=128), g=None) == binding.DR_ERR_INVALID_ARG
    bad = _prob()
    bad.gate = 4
    assert _fwd(lib, bad) == binding.DR_ERR_INVALID_ARG
    n = ctypes.c_size_t(0)
    assert lib.dr_workspace_size(ctypes.byref(_prob(gate="phase", dk=128, dv=128)), 0,
                                 ctypes.byref(n)) == binding.DR_OK and n.value > 0


def test_inject_timeout_arguments(lib):
    assert lib.dr_inject_timeout(-1) == binding.DR_ERR_INVALID_ARG
    assert lib.dr_inject_timeout(0) == binding.DR_OK
