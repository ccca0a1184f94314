"""Pins for the fp64 oracle: checks against what the pages and the mathematics
fix, never against the oracle itself.

* chunkwise form == token-by-token form in exact arithmetic (ReWY abstract,
  paperdot listing: "preserving the recurrence and gradients in exact
  arithmetic"; SFDA explainer, gist.science, "Ergebnisse": chunk-WY recursion
  and affine chunk transfer agree with brute force to 1e-10..1e-15);
* hand-derived gradients == central finite differences ("complete-gradient
  checks", ReWY abstract);
* KDA with all channels equal == GDN (SFDA explainer, "Zentrale Beiträge": KDA
  is the phase-free case; a scalar gate is a per-channel gate with equal
  channels);
* Kaczmarz step beta = eta / (||k||^2 + eps) (KLA abstract, thelatestinai.com)
  and its projection invariant S_t k_t - v_t = (1 - beta_t ||k_t||^2)(P_t k_t - v_t);
* beta = 0 freezes the state up to decay; alpha = 1 with orthogonal keys is
  plain beta-weighted linear attention; beta = 2/||k||^2 is a Householder
  reflection; linearity in (v, S0); segment splitting (affine transfer).
"""
import numpy as np
import pytest

import oracle
from oracle import chunkwise as cw


def _inputs(seed, B=1, T=9, H=2, dk=3, dv=4, gate="channel", g_mean=3.0, s0=0.3,
            normalize_k=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if normalize_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    if gate == "channel":
        g = -np.log1p(np.exp(-(rng.standard_normal((B, T, H, dk)) + g_mean)))
    elif gate == "scalar":
        g = -np.log1p(np.exp(-(rng.standard_normal((B, T, H)) + g_mean)))
    else:
        g = None
    S0 = rng.standard_normal((B, H, dv, dk)) * s0 if s0 else None
    dO = rng.standard_normal((B, T, H, dv))
    dST = rng.standard_normal((B, H, dv, dk))
    return dict(q=q, k=k, v=v, beta=beta, g=g, S0=S0, dO=dO, dST=dST)


def _rel(x, y):
    return float(np.max(np.abs(x - y)) / max(np.max(np.abs(y)), 1e-300))


GATES = ["none", "scalar", "channel"]
MODES = [oracle.BETA_DIRECT, oracle.BETA_KACZMARZ]


@pytest.mark.parametrize("gate", GATES)
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("C,T", [(1, 7), (4, 18), (16, 37), (64, 70), (64, 128)])
def test_chunkwise_equals_recurrent(gate, mode, C, T):
    x = _inputs(10 + C + T, T=T, dk=5, dv=4, gate=gate, normalize_k=(mode == 0))
    args = (x["q"], x["k"], x["v"], x["beta"], x["g"], x["S0"])
    o_r, ST_r = oracle.recurrent_fwd(*args, beta_mode=mode)
    o_c, ST_c = cw.chunk_fwd(*args, C=C, beta_mode=mode)
    assert _rel(o_c, o_r) < 1e-10
    assert _rel(ST_c, ST_r) < 1e-10
    g_r = oracle.recurrent_bwd(*args, x["dO"], x["dST"], beta_mode=mode)
    g_c = cw.chunk_bwd(*args, x["dO"], x["dST"], C=C, beta_mode=mode)
    for name in ("dq", "dk", "dv", "dbeta", "dS0") + (("dg",) if gate != "none" else ()):
        assert _rel(g_c[name], g_r[name]) < 1e-10, name


def _loss(x, mode, eps):
    o, ST = oracle.recurrent_fwd(x["q"], x["k"], x["v"], x["beta"], x["g"], x["S0"],
                                 beta_mode=mode, eps=eps)
    return float(np.sum(o * x["dO"]) + np.sum(ST * x["dST"]))


@pytest.mark.parametrize("gate", GATES)
@pytest.mark.parametrize("mode", MODES)
def test_backward_matches_finite_differences(gate, mode):
    eps = 1e-6
    x = _inputs(3, T=8, dk=3, dv=4, gate=gate, normalize_k=(mode == 0))
    grads = oracle.recurrent_bwd(x["q"], x["k"], x["v"], x["beta"], x["g"], x["S0"],
                                 x["dO"], x["dST"], beta_mode=mode, eps=eps)
    h = 1e-6
    pairs = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta"), ("S0", "dS0")]
    if gate != "none":
        pairs.append(("g", "dg"))
    for name, gname in pairs:
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


def test_equal_channel_gate_is_scalar_gate():
    x = _inputs(5, T=21, dk=4, dv=3, gate="scalar")
    gch = np.repeat(x["g"][..., None], 4, axis=-1)
    a = (x["q"], x["k"], x["v"], x["beta"])
    o_s, ST_s = oracle.recurrent_fwd(*a, x["g"], x["S0"])
    o_c, ST_c = oracle.recurrent_fwd(*a, gch, x["S0"])
    assert np.array_equal(o_s, o_c) and np.array_equal(ST_s, ST_c)
    gs = oracle.recurrent_bwd(*a, x["g"], x["S0"], x["dO"], x["dST"])
    gc = oracle.recurrent_bwd(*a, gch, x["S0"], x["dO"], x["dST"])
    for n in ("dq", "dk", "dv", "dbeta", "dS0"):
        assert np.array_equal(gs[n], gc[n]), n
    assert _rel(gc["dg"].sum(-1), gs["dg"]) < 1e-12


def test_kaczmarz_is_direct_with_explicit_beta():
    eps = 1e-6
    x = _inputs(6, T=15, dk=5, dv=3, gate="scalar", normalize_k=False)
    explicit = x["beta"] / (np.sum(x["k"] ** 2, axis=-1) + eps)
    o_k, ST_k = oracle.recurrent_fwd(x["q"], x["k"], x["v"], x["beta"], x["g"], x["S0"],
                                     beta_mode=oracle.BETA_KACZMARZ, eps=eps)
    o_d, ST_d = oracle.recurrent_fwd(x["q"], x["k"], x["v"], explicit, x["g"], x["S0"])
    assert _rel(o_k, o_d) < 1e-13 and _rel(ST_k, ST_d) < 1e-13
    # chain rule: d/deta = d/dbeta / (||k||^2 + eps) at the same point
    gk = oracle.recurrent_bwd(x["q"], x["k"], x["v"], x["beta"], x["g"], x["S0"], x["dO"],
                              x["dST"], beta_mode=oracle.BETA_KACZMARZ, eps=eps)
    gd = oracle.recurrent_bwd(x["q"], x["k"], x["v"], explicit, x["g"], x["S0"], x["dO"],
                              x["dST"])
    assert _rel(gk["dbeta"], gd["dbeta"] / (np.sum(x["k"] ** 2, axis=-1) + eps)) < 1e-12


@pytest.mark.parametrize("gate", GATES)
def test_kaczmarz_projection_invariant(gate):
    """With eta = 1 and eps = 0 the Kaczmarz step makes S_t interpolate (k_t, v_t);
    for general eta the residual shrinks by exactly (1 - eta)."""
    x = _inputs(7, T=6, dk=4, dv=3, gate=gate, normalize_k=False)
    for t in range(1, 7):
        sl = {n: (None if x[n] is None else x[n][:, :t]) for n in ("q", "k", "v", "beta", "g")}
        ones = np.ones_like(sl["beta"])
        _, ST = oracle.recurrent_fwd(sl["q"], sl["k"], sl["v"], ones, sl["g"], x["S0"],
                                     beta_mode=oracle.BETA_KACZMARZ, eps=0.0)
        kt, vt = x["k"][:, t - 1], x["v"][:, t - 1]          # [B, H, d]
        resid = np.einsum("bhac,bhc->bha", ST, kt) - vt
        assert np.max(np.abs(resid)) < 1e-12
        # general eta: residual after = (1 - eta) * residual of the decayed state
        _, ST = oracle.recurrent_fwd(sl["q"], sl["k"], sl["v"], sl["beta"], sl["g"], x["S0"],
                                     beta_mode=oracle.BETA_KACZMARZ, eps=0.0)
        if t == 1:
            Sprev = x["S0"]
        else:
            _, Sprev = oracle.recurrent_fwd(*(None if a is None else a[:, : t - 1] for a in
                                              (x["q"], x["k"], x["v"], x["beta"], x["g"])),
                                            x["S0"], beta_mode=oracle.BETA_KACZMARZ, eps=0.0)
        if gate == "none":
            alpha = np.ones(kt.shape)
        elif gate == "scalar":
            alpha = np.repeat(np.exp(x["g"][:, t - 1])[..., None], kt.shape[-1], -1)
        else:
            alpha = np.exp(x["g"][:, t - 1])
        before = np.einsum("bhac,bhc->bha", Sprev * alpha[:, :, None, :], kt) - vt
        after = np.einsum("bhac,bhc->bha", ST, kt) - vt
        eta = x["beta"][:, t - 1][..., None]
        assert np.max(np.abs(after - (1 - eta) * before)) < 1e-12


@pytest.mark.parametrize("gate", GATES)
def test_beta_zero_freezes_state_up_to_decay(gate):
    x = _inputs(8, T=11, dk=4, dv=3, gate=gate)
    zero = np.zeros_like(x["beta"])
    o, ST = oracle.recurrent_fwd(x["q"], x["k"], x["v"], zero, x["g"], x["S0"])
    B, T, H, dk = x["q"].shape
    if gate == "none":
        cum = np.zeros((B, T, H, dk))
    elif gate == "scalar":
        cum = np.repeat(np.cumsum(x["g"], axis=1)[..., None], dk, -1)
    else:
        cum = np.cumsum(x["g"], axis=1)
    # o_t = S0 Gamma_t q_t with Gamma_t = Diag(exp(sum_{s<=t} g_s))
    expect = np.einsum("bhac,bthc->btha", x["S0"], np.exp(cum) * x["q"])
    assert _rel(o, expect) < 1e-13
    assert _rel(ST, x["S0"] * np.exp(cum[:, -1])[:, :, None, :]) < 1e-13


def test_orthogonal_keys_give_linear_attention():
    """alpha = 1, S0 = 0 and mutually orthogonal keys: every erase sees an empty
    direction, so o_t = sum_{j<=t} beta_j (k_j . q_t) v_j exactly."""
    rng = np.random.default_rng(9)
    T, dk, dv = 6, 8, 5
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = (Qm[:T] * rng.uniform(0.5, 2.0, size=(T, 1)))[None, :, None, :]
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    beta = rng.uniform(0.1, 0.9, size=(1, T, 1))
    o, _ = oracle.recurrent_fwd(q, k, v, beta)
    scores = np.tril(q[0, :, 0] @ k[0, :, 0].T) * beta[0, :, 0][None, :]
    expect = scores @ v[0, :, 0]
    assert _rel(o[0, :, 0], expect) < 1e-13


def test_householder_step_is_a_reflection():
    """alpha = 1, v = 0, beta_t = 2/||k_t||^2: each step right-multiplies the state
    by the Householder reflection I - 2 k k^T/||k||^2."""
    rng = np.random.default_rng(11)
    T, dk, dv = 5, 4, 3
    k = rng.standard_normal((1, T, 1, dk))
    beta = 2.0 / np.sum(k ** 2, axis=-1)
    S0 = rng.standard_normal((1, 1, dv, dk))
    _, ST = oracle.recurrent_fwd(rng.standard_normal((1, T, 1, dk)), k,
                                 np.zeros((1, T, 1, dv)), beta, None, S0)
    Hprod = np.eye(dk)
    for t in range(T):
        kt = k[0, t, 0]
        Hprod = Hprod @ (np.eye(dk) - 2.0 * np.outer(kt, kt) / (kt @ kt))
    assert _rel(ST[0, 0], S0[0, 0] @ Hprod) < 1e-13
    assert abs(np.linalg.norm(ST) - np.linalg.norm(S0)) < 1e-12


def test_linear_in_values_and_initial_state():
    x = _inputs(12, T=10, dk=3, dv=4, gate="channel")
    y = _inputs(13, T=10, dk=3, dv=4, gate="channel")
    a, b = 0.7, -1.3
    base = (x["q"], x["k"])
    o1, S1 = oracle.recurrent_fwd(*base, x["v"], x["beta"], x["g"], x["S0"])
    o2, S2 = oracle.recurrent_fwd(*base, y["v"], x["beta"], x["g"], y["S0"])
    o3, S3 = oracle.recurrent_fwd(*base, a * x["v"] + b * y["v"], x["beta"], x["g"],
                                  a * x["S0"] + b * y["S0"])
    assert _rel(o3, a * o1 + b * o2) < 1e-12 and _rel(S3, a * S1 + b * S2) < 1e-12


@pytest.mark.parametrize("gate", GATES)
def test_segment_split_is_exact(gate):
    """Affine chunk transfer: running [0, T) equals running [0, T1) and then
    [T1, T) from the carried state, forward and backward."""
    x = _inputs(14, T=23, dk=4, dv=3, gate=gate)
    T1 = 9

    def part(a, lo, hi):
        return None if a is None else a[:, lo:hi]

    names = ("q", "k", "v", "beta", "g")
    o, ST = oracle.recurrent_fwd(*(x[n] for n in names), x["S0"])
    oa, Sa = oracle.recurrent_fwd(*(part(x[n], 0, T1) for n in names), x["S0"])
    ob, Sb = oracle.recurrent_fwd(*(part(x[n], T1, 23) for n in names), Sa)
    assert _rel(np.concatenate([oa, ob], axis=1), o) < 1e-13 and _rel(Sb, ST) < 1e-13
    full = oracle.recurrent_bwd(*(x[n] for n in names), x["S0"], x["dO"], x["dST"])
    gb = oracle.recurrent_bwd(*(part(x[n], T1, 23) for n in names), Sa,
                              part(x["dO"], T1, 23), x["dST"])
    ga = oracle.recurrent_bwd(*(part(x[n], 0, T1) for n in names), x["S0"],
                              part(x["dO"], 0, T1), gb["dS0"])
    for n in ("dq", "dk", "dv", "dbeta") + (("dg",) if gate != "none" else ()):
        assert _rel(np.concatenate([ga[n], gb[n]], axis=1), full[n]) < 1e-12, n
    assert _rel(ga["dS0"], full["dS0"]) < 1e-12


def test_long_sequence_checkpointing_consistent():
    """The backward re-runs segments from checkpoints whose spacing grows with T
    (64 tokens, doubled past T = 4096); T = 5000 uses 128-token segments and
    must still agree with the chunkwise restatement."""
    x = _inputs(15, T=5000, H=1, dk=3, dv=2, gate="scalar")
    names = ("q", "k", "v", "beta", "g")
    full = oracle.recurrent_bwd(*(x[n] for n in names), x["S0"], x["dO"], x["dST"])
    chunk = cw.chunk_bwd(*(x[n] for n in names), x["S0"], x["dO"], x["dST"], C=32)
    for n in ("dq", "dk", "dv", "dbeta", "dg", "dS0"):
        assert _rel(chunk[n], full[n]) < 1e-10, n
