"""Pins for the oracle's phase (SFDA rotation-decay) gate, against what the
SFDA explainer ("Semidirect Fourier Delta Attention", gist.science) and the
mathematics fix -- never against the oracle's own formulas:

* the page's update in complex coordinates, Lambda_t = diag(alpha_t e^{i theta_t})
  ("Kernarchitektur"): with no write (beta = 0) the state's complex key
  coordinates z = x + i y are multiplied by prod_t alpha_t e^{i theta_t},
  evaluated here with numpy's complex arithmetic;
* zero phase recovers KDA ("SFDA ... enthält KDA als Spezialfall"; "KDA
  zurückgewinnt, wenn die Phasen Null sind"), both channels of a pair sharing
  the decay -- the per-channel path is pinned on its own;
* the phase-only cyclic counter ("Perfekte Zähler", mod-5 counter): with
  theta = 2 pi / 5 and alpha = 1 the decay is the identity after five tokens,
  and a rotation keeps the state's norm;
* the delta rule's write lands exactly whatever the decay: with
  beta = 1 / ||k||^2 the new state maps k_t to v_t, which fixes that the
  rotation acts before the erase-and-write ("(I - beta k k^*) Lambda_t S");
* the hand-derived gradients (including d/d log alpha and d/d theta) against
  central finite differences;
* the chunk recursion with rotation-decay factors equals the token-by-token
  result ("Konstruktives Chunk-WY-Theorem"; "Ergebnisse": the formulas agree
  with brute force), for chunk sizes 1 to 64 and ragged tails.
"""
import numpy as np
import pytest

import oracle


def _phase_inputs(seed, B=1, T=7, H=2, dk=4, dv=3, s0=0.5, theta_scale=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    g = np.zeros((B, T, H, dk))
    g[..., 0::2] = -np.log1p(np.exp(-(rng.standard_normal((B, T, H, dk // 2)) + 2.0)))
    g[..., 1::2] = theta_scale * rng.uniform(-np.pi, np.pi, (B, T, H, dk // 2))
    S0 = rng.standard_normal((B, H, dv, dk)) * s0
    dO = rng.standard_normal((B, T, H, dv))
    dST = rng.standard_normal((B, H, dv, dk))
    return dict(q=q, k=k, v=v, beta=beta, g=g, S0=S0, dO=dO, dST=dST)


def _rel(x, y):
    return float(np.max(np.abs(x - y)) / max(np.max(np.abs(y)), 1e-300))


def _fwd(x, **kw):
    return oracle.recurrent_fwd(x["q"], x["k"], x["v"], x["beta"], x["g"], x["S0"],
                                gate=oracle.GATE_PHASE, **kw)


def test_no_write_is_complex_diagonal_product():
    x = _phase_inputs(1, T=9, dk=6, dv=4)
    x["beta"][:] = 0.0
    o, ST = _fwd(x)
    # complex key coordinates of every state row: z_j = S[:, 2j] + i S[:, 2j+1]
    z = x["S0"][..., 0::2] + 1j * x["S0"][..., 1::2]            # [B, H, dv, dk/2]
    lam = np.exp(x["g"][..., 0::2]) * np.exp(1j * x["g"][..., 1::2])  # [B, T, H, dk/2]
    B, T, H = x["beta"].shape
    for t in range(T):
        z = z * lam[:, t][:, :, None, :]
        S_t = np.empty_like(x["S0"])
        S_t[..., 0::2], S_t[..., 1::2] = z.real, z.imag
        o_t = np.einsum("bhac,bhc->bha", S_t, x["q"][:, t])
        assert _rel(o[:, t], o_t) < 1e-13
    assert _rel(ST, S_t) < 1e-13


@pytest.mark.parametrize("mode", [oracle.BETA_DIRECT, oracle.BETA_KACZMARZ])
def test_zero_phase_is_kda_with_paired_decay(mode):
    x = _phase_inputs(2, T=11, dk=6, dv=5)
    x["g"][..., 1::2] = 0.0
    g_kda = x["g"].copy()
    g_kda[..., 1::2] = x["g"][..., 0::2]       # both channels of a pair decay alike
    o_p, S_p = _fwd(x, beta_mode=mode)
    o_k, S_k = oracle.recurrent_fwd(x["q"], x["k"], x["v"], x["beta"], g_kda, x["S0"],
                                    beta_mode=mode)
    assert _rel(o_p, o_k) < 1e-14 and _rel(S_p, S_k) < 1e-14
    gp = oracle.recurrent_bwd(x["q"], x["k"], x["v"], x["beta"], x["g"], x["S0"], x["dO"],
                              x["dST"], beta_mode=mode, gate=oracle.GATE_PHASE)
    gk = oracle.recurrent_bwd(x["q"], x["k"], x["v"], x["beta"], g_kda, x["S0"], x["dO"],
                              x["dST"], beta_mode=mode)
    for n in ("dq", "dk", "dv", "dbeta", "dS0"):
        assert _rel(gp[n], gk[n]) < 1e-13, n
    # d/d log alpha_j of the tied decay is the sum of the two channels' gradients
    assert _rel(gp["dg"][..., 0::2], gk["dg"][..., 0::2] + gk["dg"][..., 1::2]) < 1e-13


def test_mod5_phase_counter_is_exactly_periodic():
    # alpha = 1, theta = 2 pi / 5 on every pair, no writes: period five
    x = _phase_inputs(3, T=20, dk=8, dv=3)
    x["beta"][:] = 0.0
    x["g"][..., 0::2] = 0.0
    x["g"][..., 1::2] = 2.0 * np.pi / 5.0
    x["q"][:] = x["q"][:, :1]                  # the same query at every token
    o, ST = _fwd(x)
    assert _rel(ST, x["S0"]) < 1e-13           # 20 tokens = four full turns
    assert _rel(o[:, 5:], o[:, :-5]) < 1e-13
    assert _rel(o[:, 1], o[:, 0]) > 1e-2       # but not period one
    # a rotation keeps every state row's norm
    x["g"][..., 1::2] = np.random.default_rng(4).uniform(-3, 3, x["g"][..., 1::2].shape)
    _, ST = _fwd(x)
    assert _rel(np.linalg.norm(ST, axis=-1), np.linalg.norm(x["S0"], axis=-1)) < 1e-13


def test_write_lands_after_rotation():
    # beta_t = 1 / ||k_t||^2 (Kaczmarz with eta = 1, eps = 0): S_t k_t = v_t exactly
    x = _phase_inputs(5, T=1, dk=6, dv=4)
    x["k"] = x["k"] * 1.7
    x["beta"][:] = 1.0
    o, ST = _fwd(x, beta_mode=oracle.BETA_KACZMARZ, eps=0.0)
    Sk = np.einsum("bhac,bhc->bha", ST, x["k"][:, 0])
    assert _rel(Sk, x["v"][:, 0]) < 1e-13
    # and the erased state agrees with the rotated S0 off the key direction
    z = (x["S0"][..., 0::2] + 1j * x["S0"][..., 1::2]) * \
        (np.exp(x["g"][:, 0, :, 0::2]) * np.exp(1j * x["g"][:, 0, :, 1::2]))[:, :, None, :]
    P = np.empty_like(x["S0"])
    P[..., 0::2], P[..., 1::2] = z.real, z.imag
    kk = x["k"][:, 0] / np.linalg.norm(x["k"][:, 0], axis=-1, keepdims=True)
    perp = np.random.default_rng(6).standard_normal(kk.shape)
    perp -= np.sum(perp * kk, axis=-1, keepdims=True) * kk
    assert _rel(np.einsum("bhac,bhc->bha", ST, perp),
                np.einsum("bhac,bhc->bha", P, perp)) < 1e-12


def _loss(x, mode, eps):
    o, ST = _fwd(x, beta_mode=mode, eps=eps)
    return float(np.sum(o * x["dO"]) + np.sum(ST * x["dST"]))


@pytest.mark.parametrize("mode", [oracle.BETA_DIRECT, oracle.BETA_KACZMARZ])
def test_phase_backward_matches_finite_differences(mode):
    eps = 1e-6
    x = _phase_inputs(7, T=6, dk=4, dv=3)
    grads = oracle.recurrent_bwd(x["q"], x["k"], x["v"], x["beta"], x["g"], x["S0"],
                                 x["dO"], x["dST"], beta_mode=mode, eps=eps,
                                 gate=oracle.GATE_PHASE)
    h = 1e-6
    for name, gname in [("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta"),
                        ("S0", "dS0"), ("g", "dg")]:
        base = x[name]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            keep = base[idx]
            base[idx] = keep + h
            lp = _loss(x, mode, eps)
            base[idx] = keep - h
            lm = _loss(x, mode, eps)
            base[idx] = keep
            fd[idx] = (lp - lm) / (2 * h)
        assert _rel(grads[gname], fd) < 1e-6, gname


def test_phase_gate_rejects_odd_key_dim():
    x = _phase_inputs(8, dk=4)
    with pytest.raises(ValueError):
        oracle.recurrent_fwd(x["q"][..., :3], x["k"][..., :3], x["v"], x["beta"],
                             x["g"][..., :3], None, gate=oracle.GATE_PHASE)


@pytest.mark.parametrize("mode", [oracle.BETA_DIRECT, oracle.BETA_KACZMARZ])
@pytest.mark.parametrize("C,T", [(1, 5), (4, 13), (16, 37), (64, 70)])
def test_phase_chunkwise_equals_recurrent(mode, C, T):
    # "Konstruktives Chunk-WY-Theorem" and the brute-force agreement of
    # "Ergebnisse": the chunk recursion with the rotation-decay reaches the
    # token-by-token result exactly (up to rounding)
    from oracle import chunkwise as cw
    x = _phase_inputs(20 + C + T, T=T, dk=6, dv=4, theta_scale=1.0)
    if mode == oracle.BETA_KACZMARZ:
        x["k"] = x["k"] * 1.3
    o_r, S_r = _fwd(x, beta_mode=mode)
    o_c, S_c = cw.chunk_fwd_phase(x["q"], x["k"], x["v"], x["beta"], x["g"], x["S0"], C=C,
                                  beta_mode=mode)
    assert _rel(o_c, o_r) < 1e-10 and _rel(S_c, S_r) < 1e-10


@pytest.mark.parametrize("mode", [oracle.BETA_DIRECT, oracle.BETA_KACZMARZ])
@pytest.mark.parametrize("C,T", [(1, 5), (4, 13), (16, 37), (64, 70)])
def test_phase_chunkwise_backward_equals_recurrent(mode, C, T):
    # the residual-system backward of the chunk form with rotation-decay
    # factors reaches the token-by-token gradients, d/d log alpha and d/d theta
    # included (the same exactness claim, for the gradients)
    from oracle import chunkwise as cw
    x = _phase_inputs(40 + C + T, T=T, dk=6, dv=4)
    if mode == oracle.BETA_KACZMARZ:
        x["k"] = x["k"] * 1.3
    args = (x["q"], x["k"], x["v"], x["beta"], x["g"], x["S0"], x["dO"], x["dST"])
    g_r = oracle.recurrent_bwd(*args, beta_mode=mode, gate=oracle.GATE_PHASE)
    g_c = cw.chunk_bwd_phase(*args, C=C, beta_mode=mode)
    for name in ("dq", "dk", "dv", "dbeta", "dg", "dS0"):
        assert _rel(g_c[name], g_r[name]) < 1e-9, name
