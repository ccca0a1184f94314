"""GPU parity of the single-token decode step (dr_decode_step) against the fp64
oracle's token-by-token recurrence: one step from a random state, and a run of
steps whose state is carried between calls.  Bars: the fp32 state to 1e-4
relative (it is computed in fp32 from the same inputs), o to 1e-4 for fp32
storage and 2e-2 for bf16 storage (o is rounded to bf16)."""
import numpy as np
import pytest
import torch

import oracle
from _parity import rel_err
from delta_rule_linear_chunkwise_b200 import WORKLOADS, binding, make_inputs
from delta_rule_linear_chunkwise_b200.workloads import random_state

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    binding.load()


def _mode(w):
    return oracle.BETA_KACZMARZ if w.beta_mode == "kaczmarz" else oracle.BETA_DIRECT


def _run(w, steps, s0_seed=21):
    """`steps` decode calls on the GPU vs the oracle's recurrence over the same
    tokens.  Returns (o error, final state error)."""
    inp = make_inputs(w.with_(T=steps))
    S0 = random_state(w, seed=s0_seed, std=0.3)
    o_ref, ST_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"],
                                         S0, beta_mode=_mode(w), eps=w.eps)
    S = S0.clone().cuda()
    outs = []
    for t in range(steps):
        sl = lambda x: None if x is None else x[:, t:t + 1].contiguous().cuda()
        outs.append(binding.decode_step(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["beta"]),
                                        sl(inp["g"]), S, beta_mode=w.beta_mode, eps=w.eps))
    torch.cuda.synchronize()
    assert binding.last_device_error() == binding.DR_OK
    o = torch.cat(outs, dim=1).float().cpu().numpy()
    return rel_err(o, o_ref), rel_err(S.cpu().numpy(), ST_ref)


CASES = [
    ("kda_bf16_b4h16t8192", {}),
    ("gdn_bf16_b4h8t2048", {}),
    ("deltanet_bf16_b4h8t2048", {}),
    ("kla_bf16_b1h16t65536", {}),
    ("kda_bf16_b4h16t8192", {"dtype": "f32"}),
    ("kla_bf16_b1h16t65536", {"dtype": "f32"}),
    ("gdn_f32_b1h2t256d64", {}),
    ("kda_bf16_b4h16t8192", {"dk": 64, "dv": 32}),
    ("kda_bf16_b4h16t8192", {"dk": 16, "dv": 16, "dtype": "f32"}),
]


@pytest.mark.parametrize("name,kw", CASES, ids=[f"{n}-{'-'.join(f'{k}{v}' for k, v in kw.items())}"
                                               for n, kw in CASES])
def test_decode_single_step(name, kw):
    w = WORKLOADS[name].with_(name="dec", B=3, H=5, **kw)
    eo, es = _run(w, 1)
    assert es <= 1e-4, es
    assert eo <= (1e-4 if w.dtype == "f32" else 2e-2), eo


@pytest.mark.parametrize("name", ["kda_bf16_b4h16t8192", "kla_bf16_b1h16t65536"])
def test_decode_carries_state_over_steps(name):
    w = WORKLOADS[name].with_(name="dec_run", B=2, H=3)
    eo, es = _run(w, 40)
    assert es <= 1e-4, es
    assert eo <= 2e-2, eo


def test_decode_large_batch_sampled():
    """A serving-sized batch (B = 64, H = 16), compared on a few heads."""
    w = WORKLOADS["kda_bf16_b4h16t8192"].with_(name="dec_big", B=64, H=16, T=1)
    inp = make_inputs(w)
    S0 = random_state(w, seed=22, std=0.3)
    S = S0.clone().cuda()
    o = binding.decode_step(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(),
                            inp["beta"].cuda(), inp["g"].cuda(), S)
    torch.cuda.synchronize()
    o = o.float().cpu().numpy()
    S = S.cpu().numpy()
    for b, h in [(0, 0), (31, 7), (63, 15)]:
        pick = lambda x: None if x is None else x[b:b + 1, :, h:h + 1]
        o_ref, ST_ref = oracle.recurrent_fwd(pick(inp["q"]), pick(inp["k"]), pick(inp["v"]),
                                             pick(inp["beta"]), pick(inp["g"]),
                                             S0[b:b + 1, h:h + 1], eps=w.eps)
        assert rel_err(S[b, h], ST_ref[0, 0]) <= 1e-4
        assert rel_err(o[b, 0, h], o_ref[0, 0, 0]) <= 2e-2
