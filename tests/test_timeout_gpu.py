"""The bounded-wait timeout path, driven without faulting the GPU.

dr_inject_timeout makes the next chunk-backward launch wait, with a short
limit, on an mbarrier that nothing arrives on (after its inputs have landed and
before it issues any tensor-core instruction).  The wait must give up, the call
must return, dr_last_device_error must report DR_ERR_TIMEOUT once, and the
next, uninjected call must run normally and meet the parity bar."""
import time

import pytest
import torch

from _parity import compare, run_gpu, run_oracle, select, tol
from delta_rule_linear_chunkwise_b200 import WORKLOADS, binding, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    binding.load()


def test_injected_wait_times_out_and_the_context_stays_usable():
    w = WORKLOADS["kda_bf16_b4h16t8192"].with_(name="timeout", B=1, H=2, T=200, s0_std=0.1)
    inp = make_inputs(w)
    plan = binding.Plan.for_workload(w)
    d = {n: (None if x is None else x.cuda()) for n, x in inp.items()}
    o, ST, saved = plan.fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"])
    torch.cuda.synchronize()
    assert binding.last_device_error() == binding.DR_OK
    try:
        binding.inject_timeout(1)
        t0 = time.perf_counter()
        plan.bwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], d["dO"], None, saved)
        status = binding.last_device_error()          # synchronises the stream
        elapsed = time.perf_counter() - t0
    finally:
        binding.inject_timeout(0)
    assert status == binding.DR_ERR_TIMEOUT
    assert elapsed < 30.0
    # the flag was cleared by the read, and the context still works
    assert binding.last_device_error() == binding.DR_OK
    gpu = run_gpu(w, inp)
    ref, heads = run_oracle(w, inp, None)
    errs = compare(w, select(gpu, heads), ref)
    assert all(e <= tol(w) for e in errs.values()), errs
