"""dr_chunk_fwd_static: the forward for callers that cannot allocate device
memory (and so cannot pass a workspace) runs on the library's built-in static
scratch.  Its results must match dr_chunk_fwd with a caller-provided
workspace, call after call, although every call reuses the same scratch.

This file is collected last, so a run that stops at the first failure has
already run every other test."""
import ctypes

import pytest
import torch

from delta_rule_linear_chunkwise_b200 import WORKLOADS, binding, make_inputs

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 64 << 20  # DR_STATIC_SCRATCH_BYTES in include/dr.h


def _lib():
    lib = binding.load()
    f = lib.dr_chunk_fwd_static
    f.argtypes = [ctypes.POINTER(binding.DrProblem)] + [ctypes.c_void_p] * 9
    f.restype = ctypes.c_int
    return lib


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


# Two problems: a short one (plain sequential scans) and a long one with few
# heads, which takes the chunk-parallel affine scan and so also keeps segment
# transfer matrices and states in the static scratch.
CASES = [
    WORKLOADS["kda_bf16_b4h16t8192"].with_(name="noalloc", B=2, H=4, T=1000, s0_std=0.1),
    WORKLOADS["kda_bf16_b4h16t8192"].with_(name="noalloc_segmented", B=1, H=2, T=4096,
                                           s0_std=0.1),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_static_scratch_forward_matches_workspace_forward_twice(w):
    """Both entry points run the same kernels on the same inputs, so their
    results must be bit-identical; two calls in a row with different inputs
    check that nothing left in the shared scratch by one call leaks into the
    next."""
    lib = _lib()
    plan = binding.Plan.for_workload(w)
    assert binding.workspace_size(plan.prob, 0) <= STATIC_SCRATCH_BYTES
    stream = torch.cuda.current_stream()
    for seed in (11, 12):                     # two calls in a row, different inputs
        d = {n: (None if x is None else x.cuda()) for n, x in make_inputs(w, seed=seed).items()}
        o_ref, ST_ref, _ = plan.fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"],
                                    save=False)
        o = torch.empty_like(o_ref)
        ST = torch.empty_like(ST_ref)
        ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
        st = lib.dr_chunk_fwd_static(ctypes.byref(plan.prob), ptr(d["q"]), ptr(d["k"]),
                                     ptr(d["v"]), ptr(d["beta"]), ptr(d["g"]), ptr(d["S0"]),
                                     ptr(o), ptr(ST), ctypes.c_void_p(stream.cuda_stream))
        assert st == binding.DR_OK, binding.status_string(st)
        torch.cuda.synchronize()
        assert binding.last_device_error() == binding.DR_OK
        assert torch.isfinite(o.float()).all() and torch.isfinite(ST).all()
        assert torch.equal(o, o_ref)
        assert torch.equal(ST, ST_ref)


def test_static_scratch_rejects_problems_beyond_its_size():
    lib = _lib()
    big = binding.make_problem(4, 16, 8192, 128, 128, gate="channel")
    assert binding.workspace_size(big, 0) > STATIC_SCRATCH_BYTES
    t = torch.empty(16, device="cuda")
    p = ctypes.c_void_p(t.data_ptr())
    st = lib.dr_chunk_fwd_static(ctypes.byref(big), p, p, p, p, p, None, p, None, None)
    assert st == binding.DR_ERR_WORKSPACE
