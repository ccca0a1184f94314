"""GPU parity of the SFDA phase gate (2 x 2 rotation-decay per key pair) against
the fp64 oracle's token-by-token recurrence with the same gate and its
hand-derived backward: the chunkwise forward on the tensor-core path (o and the
final state), the chunkwise backward (dq, dk, dv, dbeta, d log alpha and d theta,
dS0), and the decode step.  Bar: 2e-2 max relative error for bf16 storage (the
chunk tiles are bf16 operands with fp32 accumulation); the decode step's fp32
state to 1e-4 and its fp32 output to 1e-4."""
import numpy as np
import pytest
import torch

import oracle
from _parity import compare, rel_err, run_gpu, run_oracle, select, tol
from delta_rule_linear_chunkwise_b200 import WORKLOADS, binding, make_inputs
from delta_rule_linear_chunkwise_b200.workloads import random_state

pytestmark = pytest.mark.gpu

SFDA = WORKLOADS["sfda_bf16_b4h16t8192"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    binding.load()


def _mode(w):
    return oracle.BETA_KACZMARZ if w.beta_mode == "kaczmarz" else oracle.BETA_DIRECT


def _fwd_check(w, heads=None, save=False):
    inp = make_inputs(w)
    plan = binding.Plan.for_workload(w)
    d = {n: (None if x is None else x.cuda()) for n, x in inp.items()}
    o, ST, _ = plan.fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], save=save)
    torch.cuda.synchronize()
    assert binding.last_device_error() == binding.DR_OK
    o, ST = o.float().cpu().numpy(), ST.cpu().numpy()
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    errs = []
    for b, h in heads:
        pick = lambda x: None if x is None else x[b:b + 1, :, h:h + 1].double().numpy()
        S0 = None if inp["S0"] is None else inp["S0"][b:b + 1, h:h + 1].double().numpy()
        o_ref, ST_ref = oracle.recurrent_fwd(pick(inp["q"]), pick(inp["k"]), pick(inp["v"]),
                                             pick(inp["beta"]), pick(inp["g"]), S0,
                                             beta_mode=_mode(w), eps=w.eps,
                                             gate=oracle.GATE_PHASE)
        errs.append((rel_err(o[b, :, h], o_ref[0, :, 0]), rel_err(ST[b, h], ST_ref[0, 0])))
    eo, es = max(e[0] for e in errs), max(e[1] for e in errs)
    assert eo <= 2e-2 and es <= 2e-2, f"{w.name}: o {eo:.2e}, S_T {es:.2e}"
    return eo, es


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 129, 200])
def test_sfda_forward_ragged_all_heads(T):
    _fwd_check(SFDA.with_(name=f"sfda_t{T}", B=2, H=3, T=T, s0_std=0.1))


def test_sfda_forward_saving_and_kaczmarz():
    _fwd_check(SFDA.with_(name="sfda_save", B=1, H=2, T=300, s0_std=0.1), save=True)
    _fwd_check(SFDA.with_(name="sfda_kacz", B=1, H=2, T=300, beta_mode="kaczmarz",
                          normalize_k=False, s0_std=0.1))


def test_sfda_forward_strong_decay_and_large_phase():
    # decays near e^{-1.3} per token and phases up to pi: the centred factors
    # and the accumulated in-chunk phase stay in range
    _fwd_check(SFDA.with_(name="sfda_strong", B=1, H=2, T=256, g_mean=-1.0, s0_std=0.1))


@pytest.mark.parametrize("T", [4096, 4096 + 100])
def test_sfda_segmented_affine_scan(T):
    # few heads, many chunks: the forward runs the chunk-parallel segmented scan
    _fwd_check(SFDA.with_(name=f"sfda_seg{T}", B=1, H=4, T=T, s0_std=0.1),
               heads=[(0, 0), (0, 3)])


def test_sfda_full_size_sampled_heads():
    # the benchmark's configuration (B4 H16 T8192 d128 bf16), sampled heads
    eo, es = _fwd_check(SFDA, heads=[(0, 0), (2, 7), (3, 15)], save=True)
    print(f"sfda full size: o {eo:.2e}, S_T {es:.2e}")


def test_sfda_zero_phase_matches_paired_kda():
    # with all phases zero the SFDA forward is KDA with each pair's decay shared
    w = SFDA.with_(name="sfda_zero", B=1, H=2, T=200, s0_std=0.1)
    inp = make_inputs(w)
    g = inp["g"].clone()
    g[..., 1::2] = 0.0
    gk = g.clone()
    gk[..., 1::2] = g[..., 0::2]
    d = {n: (None if x is None else x.cuda()) for n, x in inp.items()}
    o_p, S_p, _ = binding.Plan.for_workload(w).fwd(d["q"], d["k"], d["v"], d["beta"],
                                                   g.cuda(), d["S0"], save=False)
    o_k, S_k, _ = binding.Plan.for_workload(w.with_(gate="channel")).fwd(
        d["q"], d["k"], d["v"], d["beta"], gk.cuda(), d["S0"], save=False)
    torch.cuda.synchronize()
    assert rel_err(o_p.float().cpu().numpy(), o_k.float().cpu().numpy()) < 1e-2
    assert rel_err(S_p.cpu().numpy(), S_k.cpu().numpy()) < 1e-2


def _bwd_check(w, heads=None, save=True, dST=True):
    inp = make_inputs(w)
    dst = random_state(w, seed=41, std=0.5) if dST else None
    gpu = run_gpu(w, inp, dST=dst, save=save)
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    ref, heads = run_oracle(w, inp, heads, dST=dst)
    errs = compare(w, select(gpu, heads), ref)
    bad = {n: e for n, e in errs.items() if not (e <= tol(w))}
    assert not bad, f"{w.name}: {errs}"
    return errs


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_sfda_backward_ragged_all_heads(T):
    _bwd_check(SFDA.with_(name=f"sfda_bwd_t{T}", B=2, H=3, T=T, s0_std=0.1))


def test_sfda_backward_recompute_and_kaczmarz():
    _bwd_check(SFDA.with_(name="sfda_bwd_rec", B=1, H=2, T=300, s0_std=0.1), save=False)
    _bwd_check(SFDA.with_(name="sfda_bwd_kacz", B=1, H=2, T=300, beta_mode="kaczmarz",
                          normalize_k=False, s0_std=0.1))


@pytest.mark.parametrize("mu", [-1.0, -3.0])
def test_sfda_backward_strong_decay(mu):
    _bwd_check(SFDA.with_(name=f"sfda_bwd_strong{mu}", B=1, H=2, T=256, g_mean=mu,
                          s0_std=0.3))


def test_sfda_backward_segmented_affine_scan():
    _bwd_check(SFDA.with_(name="sfda_bwd_seg", B=1, H=2, T=4096 + 100, s0_std=0.1))


def test_sfda_backward_full_size_sampled_heads():
    errs = _bwd_check(SFDA, heads=[(0, 0), (2, 7), (3, 15)], dST=False)
    print("sfda backward full size", {k: f"{v:.2e}" for k, v in errs.items()})


def test_sfda_zero_phase_backward_matches_paired_kda():
    # zero phase: the SFDA backward is KDA's with each pair's decay shared, and
    # d/d log alpha of a pair is the sum of its two channels' KDA gradients
    w = SFDA.with_(name="sfda_zero_bwd", B=1, H=2, T=200, s0_std=0.1)
    inp = make_inputs(w)
    g = inp["g"].clone()
    g[..., 1::2] = 0.0
    gk = g.clone()
    gk[..., 1::2] = g[..., 0::2]
    ip = dict(inp, g=g)
    ik = dict(inp, g=gk)
    a = run_gpu(w, ip)
    b = run_gpu(w.with_(gate="channel"), ik)
    for n in ("dq", "dk", "dv", "dbeta", "dS0"):
        assert rel_err(a[n], b[n]) < 1e-2, n
    assert rel_err(a["dg"][..., 0::2], b["dg"][..., 0::2] + b["dg"][..., 1::2]) < 1e-2


@pytest.mark.parametrize("kw", [{}, {"dtype": "f32"}, {"dk": 64, "dv": 32},
                                {"beta_mode": "kaczmarz", "normalize_k": False}])
def test_sfda_decode_steps(kw):
    w = SFDA.with_(B=3, H=4, **kw)
    steps = 20
    inp = make_inputs(w.with_(T=steps))
    S0 = random_state(w, seed=31, std=0.3)
    o_ref, ST_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"],
                                         S0, beta_mode=_mode(w), eps=w.eps,
                                         gate=oracle.GATE_PHASE)
    S = S0.clone().cuda()
    outs = []
    for t in range(steps):
        sl = lambda x: x[:, t:t + 1].contiguous().cuda()
        outs.append(binding.decode_step(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]),
                                        sl(inp["beta"]), sl(inp["g"]), S, gate="phase",
                                        beta_mode=w.beta_mode, eps=w.eps))
    torch.cuda.synchronize()
    assert binding.last_device_error() == binding.DR_OK
    o = torch.cat(outs, dim=1).float().cpu().numpy()
    bar_o = 1e-4 if w.dtype == "f32" else 2e-2
    assert rel_err(o, o_ref) <= bar_o
    assert rel_err(S.cpu().numpy(), ST_ref) <= 1e-4
