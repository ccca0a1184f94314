"""fp64 numpy restatement of the chunkwise (WY / UT-transform) form.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Used to pin the claim
that the chunkwise form reaches exactly the token-by-token result ("preserving
the recurrence and gradients in exact arithmetic", ReWY abstract, paperdot
listing; "Exakter Affiner Chunk-Transfer" and the brute-force residual check in
"Ergebnisse", SFDA explainer, gist.science) and to expose per-chunk
intermediates for debugging.  It is NOT what the CUDA path is compared against.

Per head, chunk n covers tokens [nC, nC + C); a ragged tail is padded with
k = q = v = 0, beta = 0, g = 0, which leaves the state untouched.  With
gamma_i the inclusive within-chunk cumulative log-gate (per channel; scalar
gates broadcast; zero without a gate):

    Kh = k e^{gamma}        Kb = k e^{-gamma}        Qh = q e^{gamma}
    Kt = k e^{gamma_C - gamma}      (gamma_C = gamma of the chunk's last row)
    A  = diag(beta) strict_tril(Kh Kb^T)           (C x C, strictly lower)
    (I + A) X = R,  X = [U' | W],  R = diag(beta) [V | Kh]      (UT transform)
    U  = U' - W S^T                                 (pseudo-values)
    O  = Qh S^T + tril(Qh Kb^T) U                   (inclusive causal mask)
    S' = S Diag(e^{gamma_C}) + U^T Kt               (affine chunk transfer)

The SFDA explainer writes the chunk's transition product as
Gamma - Y M W^* with a triangular M whose size is bounded by the chunk; here
that product is S -> S Diag(e^{gamma_C}) - (S W^T) Kt, i.e. Y = W, M = I, with
the triangular factor folded into W by the solve, and the write summary
B_chunk = U'^T Kt comes from the zero-initial-state recursion.

Backward (the residual-system reading of the ReWY abstract): the adjoint of
(I + A) X = R is one transposed triangular solve (I + A)^T Lam = dX, giving
dR = Lam and dA = -strict_tril(Lam X^T); no adjoint of the inverse is formed.
"""
from __future__ import annotations

import numpy as np

from . import BETA_KACZMARZ, _f64


def _pad_chunk(x, t0, t1, C):
    blk = x[t0:t1]
    if t1 - t0 == C:
        return blk.copy()
    out = np.zeros((C,) + x.shape[1:], dtype=np.float64)
    out[: t1 - t0] = blk
    return out


def _gamma(gc, C, dk):
    """Inclusive cumulative log-gate per row and channel, shape (C, dk)."""
    if gc is None:
        return np.zeros((C, dk))
    if gc.ndim == 1:
        gc = np.repeat(gc[:, None], dk, axis=1)
    return np.cumsum(gc, axis=0)


def _head_inputs(q, k, v, beta, g, b, h, beta_mode, eps):
    qh, kh, vh = q[b, :, h], k[b, :, h], v[b, :, h]
    eta = beta[b, :, h]
    norm = np.sum(kh * kh, axis=1)
    bt = eta / (norm + eps) if beta_mode == BETA_KACZMARZ else eta.copy()
    gh = None if g is None else g[b, :, h]
    return qh, kh, vh, eta, bt, norm, gh


def _chunk_quantities(qc, kc, vc, bc, gc, C):
    dk = kc.shape[1]
    G = _gamma(gc, C, dk)
    Kh, Kb, Qh = kc * np.exp(G), kc * np.exp(-G), qc * np.exp(G)
    Kt = kc * np.exp(G[-1][None, :] - G)
    A = bc[:, None] * np.tril(Kh @ Kb.T, -1)
    IA = np.eye(C) + A
    R = bc[:, None] * np.concatenate([vc, Kh], axis=1)
    X = np.linalg.solve(IA, R)
    dv = vc.shape[1]
    return dict(G=G, Kh=Kh, Kb=Kb, Qh=Qh, Kt=Kt, A=A, IA=IA, X=X,
                Up=X[:, :dv], W=X[:, dv:], Mm=np.tril(Qh @ Kb.T))


def chunk_fwd(q, k, v, beta, g=None, S0=None, C=64, beta_mode=0, eps=1e-6,
              return_states=False):
    """Chunkwise forward.  Returns ``(o, S_T)`` (plus per-chunk start states)."""
    q, k, v, beta, g, S0 = map(_f64, (q, k, v, beta, g, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    nc = (T + C - 1) // C
    states = np.zeros((B, H, nc, dv, dk))
    for b in range(B):
        for h in range(H):
            qh, kh, vh, _, bt, _, gh = _head_inputs(q, k, v, beta, g, b, h, beta_mode, eps)
            S = np.zeros((dv, dk)) if S0 is None else S0[b, h].copy()
            for n in range(nc):
                t0, t1 = n * C, min(T, n * C + C)
                qc, kc, vc = (_pad_chunk(x, t0, t1, C) for x in (qh, kh, vh))
                bc = _pad_chunk(bt, t0, t1, C)
                gc = None if gh is None else _pad_chunk(gh, t0, t1, C)
                z = _chunk_quantities(qc, kc, vc, bc, gc, C)
                states[b, h, n] = S
                U = z["Up"] - z["W"] @ S.T
                O = z["Qh"] @ S.T + z["Mm"] @ U
                o[b, t0:t1, h] = O[: t1 - t0]
                S = S * np.exp(z["G"][-1])[None, :] + U.T @ z["Kt"]
            ST[b, h] = S
    if return_states:
        return o, ST, states
    return o, ST


def chunk_bwd(q, k, v, beta, g, S0, dO, dST=None, C=64, beta_mode=0, eps=1e-6):
    """Chunkwise backward through the triangular residual system.

    Returns a dict ``dq, dk, dv, dbeta, dg, dS0`` with the same conventions as
    ``oracle.recurrent_bwd``.
    """
    q, k, v, beta, g, S0, dO, dST = map(_f64, (q, k, v, beta, g, S0, dO, dST))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    nc = (T + C - 1) // C
    _, _, states = chunk_fwd(q, k, v, beta, g, S0, C, beta_mode, eps, return_states=True)
    dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    db = np.zeros((B, T, H))
    dg = None if g is None else np.zeros_like(g)
    dS0 = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            qh, kh, vh, eta, bt, norm, gh = _head_inputs(q, k, v, beta, g, b, h,
                                                         beta_mode, eps)
            dS = np.zeros((dv, dk)) if dST is None else dST[b, h].copy()
            for n in reversed(range(nc)):
                t0, t1 = n * C, min(T, n * C + C)
                m = t1 - t0
                qc, kc, vc = (_pad_chunk(x, t0, t1, C) for x in (qh, kh, vh))
                bc = _pad_chunk(bt, t0, t1, C)
                gc = None if gh is None else _pad_chunk(gh, t0, t1, C)
                dOc = _pad_chunk(dO[b, :, h], t0, t1, C)
                z = _chunk_quantities(qc, kc, vc, bc, gc, C)
                S = states[b, h, n]
                G, Kh, Kb, Qh, Kt, W, Up = (z[x] for x in ("G", "Kh", "Kb", "Qh", "Kt",
                                                          "W", "Up"))
                U = Up - W @ S.T
                decay = np.exp(G[-1])
                # outputs and state transfer of this chunk
                dU = z["Mm"].T @ dOc + Kt @ dS.T
                dMm = np.tril(dOc @ U.T)
                dQh = dOc @ S + dMm @ Kb
                dKb = dMm.T @ Qh
                dKt = U @ dS
                dW = -dU @ S
                dgamC = decay * np.sum(dS * S, axis=0)
                dS_prev = dS * decay[None, :] + dOc.T @ Qh - dU.T @ W
                # triangular residual system (I + A) X = R
                Lam = np.linalg.solve(z["IA"].T, np.concatenate([dU, dW], axis=1))
                dA = -np.tril(Lam @ z["X"].T, -1)
                LamU, LamW = Lam[:, :dv], Lam[:, dv:]
                dvc = bc[:, None] * LamU
                dKh = bc[:, None] * LamW
                dbc = np.sum(LamU * vc, axis=1) + np.sum(LamW * Kh, axis=1)
                # A = diag(beta) strict_tril(Kh Kb^T)
                dbc += np.sum(dA * np.tril(Kh @ Kb.T, -1), axis=1)
                dKh += bc[:, None] * (dA @ Kb)
                dKb += dA.T @ (bc[:, None] * Kh)
                # gate scalings
                eG = np.exp(G)
                dqc = eG * dQh
                dkc = eG * dKh + dKb / eG + np.exp(G[-1][None, :] - G) * dKt
                dG = Qh * dQh + Kh * dKh - Kb * dKb - Kt * dKt
                dG[-1] += np.sum(Kt * dKt, axis=0) + dgamC
                dgc = np.cumsum(dG[::-1], axis=0)[::-1]
                if beta_mode == BETA_KACZMARZ:
                    den = _pad_chunk(norm, t0, t1, C) + eps
                    dkc += (-2.0 * bc * dbc / den)[:, None] * kc
                    dbc = dbc / den
                dq[b, t0:t1, h] = dqc[:m]
                dkk[b, t0:t1, h] = dkc[:m]
                dvv[b, t0:t1, h] = dvc[:m]
                db[b, t0:t1, h] = dbc[:m]
                if dg is not None:
                    if dg.ndim == 4:
                        dg[b, t0:t1, h] = dgc[:m]
                    else:
                        dg[b, t0:t1, h] = dgc[:m].sum(axis=1)
                dS = dS_prev
            dS0[b, h] = dS
    return dict(dq=dq, dk=dkk, dv=dvv, dbeta=db, dg=dg, dS0=dS0)


# ---------------------------------------------------------------------------
# Phase (SFDA rotation-decay) gate.  The token decay acts on a state row as
# row -> Lambda_t row, Lambda_t the direct sum over key pairs (2j, 2j+1) of
# alpha_j [[cos theta_j, -sin theta_j], [sin theta_j, cos theta_j]] ("Semidirect
# Fourier Delta Attention", gist.science explainer, "Kernarchitektur"), i.e.
# S_t = S_{t-1} Lambda_t^T (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.  The
# blocks of different tokens commute, so with Gamma_i = Lambda_1^T ... Lambda_i^T
# (within the chunk) and the de-rotated state S~_i = S_i Gamma_i^{-1}, the chunk
# is a plain delta rule with read keys Kh_i = Gamma_i k_i and write keys
# Kb_i = Gamma_i^{-T} k_i (the page's "Konstruktives Chunk-WY-Theorem": the
# phase-decay product plus the rank-one corrections stays a chunk-local
# recursion):
#     A  = diag(beta) strict_tril(Kh Kb^T),  (I + A) [U' | W] = diag(beta) [V | Kh]
#     U  = U' - W S^T,     O = Qh S^T + tril(Qh Kb^T) U,   Qh_i = Gamma_i q_i
#     S' = S Gamma_C + U^T Kt,   Kt_i = Gamma_C^T Kb_i
# Written here with explicit d_k x d_k block matrices.

def _phase_block(g_row):
    """Lambda_t (d_k x d_k) from one token's phase gate row (log alpha_j at 2j,
    theta_j at 2j+1)."""
    dk = g_row.shape[0]
    L = np.zeros((dk, dk))
    for j in range(dk // 2):
        a, th = np.exp(g_row[2 * j]), g_row[2 * j + 1]
        L[2 * j:2 * j + 2, 2 * j:2 * j + 2] = a * np.array([[np.cos(th), -np.sin(th)],
                                                             [np.sin(th), np.cos(th)]])
    return L


def chunk_fwd_phase(q, k, v, beta, g, S0=None, C=64, beta_mode=0, eps=1e-6,
                    return_states=False):
    """Chunkwise forward with the phase gate.  Returns ``(o, S_T)``."""
    q, k, v, beta, g, S0 = map(_f64, (q, k, v, beta, g, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    nc = (T + C - 1) // C
    states = np.zeros((B, H, nc, dv, dk))
    for b in range(B):
        for h in range(H):
            qh, kh, vh, _, bt, _, gh = _head_inputs(q, k, v, beta, g, b, h, beta_mode, eps)
            S = np.zeros((dv, dk)) if S0 is None else S0[b, h].copy()
            for n in range(nc):
                t0, t1 = n * C, min(T, n * C + C)
                qc, kc, vc = (_pad_chunk(x, t0, t1, C) for x in (qh, kh, vh))
                bc = _pad_chunk(bt, t0, t1, C)
                # padded rows: log alpha = 0, theta = 0 (identity decay)
                gc = _pad_chunk(gh, t0, t1, C)
                Gam = np.zeros((C, dk, dk))
                acc = np.eye(dk)
                for i in range(C):
                    acc = acc @ _phase_block(gc[i]).T
                    Gam[i] = acc
                Kh = np.einsum("icd,id->ic", Gam, kc)
                Kb = np.stack([np.linalg.solve(Gam[i].T, kc[i]) for i in range(C)])
                Qh = np.einsum("icd,id->ic", Gam, qc)
                Kt = Kb @ Gam[-1]                       # rows (Gamma_C^T Kb_i)^T
                A = bc[:, None] * np.tril(Kh @ Kb.T, -1)
                X = np.linalg.solve(np.eye(C) + A,
                                    bc[:, None] * np.concatenate([vc, Kh], axis=1))
                Up, W = X[:, :dv], X[:, dv:]
                states[b, h, n] = S
                U = Up - W @ S.T
                O = Qh @ S.T + np.tril(Qh @ Kb.T) @ U
                o[b, t0:t1, h] = O[: t1 - t0]
                S = S @ Gam[-1] + U.T @ Kt
            ST[b, h] = S
    if return_states:
        return o, ST, states
    return o, ST


def _pairs(x):
    """Real [..., d_k] -> complex [..., d_k / 2]: channel pair (2j, 2j+1) -> x + i y."""
    return x[..., 0::2] + 1j * x[..., 1::2]


def _unpairs(z):
    out = np.empty(z.shape[:-1] + (2 * z.shape[-1],))
    out[..., 0::2], out[..., 1::2] = z.real, z.imag
    return out


def chunk_bwd_phase(q, k, v, beta, g, S0, dO, dST=None, C=64, beta_mode=0, eps=1e-6):
    """Chunkwise backward with the phase gate, through the triangular residual
    system as in ``chunk_bwd``.  Returns ``dq, dk, dv, dbeta, dg, dS0`` with
    ``dg[..., 2j]`` = d/d log alpha_j and ``dg[..., 2j+1]`` = d/d theta_j.

    On a pair read as a complex number the chunk's cumulative decay is
    zeta_i = e^{gamma_i - i Theta_i} (gamma, Theta: in-chunk cumulative sums of
    log alpha and theta), and Kh = zeta k, Kb = k / conj(zeta), Qh = zeta q,
    Kt = conj(zeta_C) / conj(zeta) k, S Gamma_C = conj(zeta_C) S per row.  For
    w = c z the gradient (d/dRe + i d/dIm) maps back by conj(c), and for a real
    parameter p of w, dL/dp = Re(conj(dL/dw) dw/dp); so each transformed tile
    gives gamma gradients Re(conj(dX) X) (with the sign of its exponent) and
    Theta gradients Im(conj(dX) X).
    """
    q, k, v, beta, g, S0, dO, dST = map(_f64, (q, k, v, beta, g, S0, dO, dST))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    nc = (T + C - 1) // C
    _, _, states = chunk_fwd_phase(q, k, v, beta, g, S0, C, beta_mode, eps,
                                   return_states=True)
    dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    db = np.zeros((B, T, H))
    dg = np.zeros_like(g)
    dS0 = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            qh_, kh_, vh, _, bt, norm, gh = _head_inputs(q, k, v, beta, g, b, h, beta_mode, eps)
            dS = np.zeros((dv, dk)) if dST is None else dST[b, h].copy()
            for n in reversed(range(nc)):
                t0, t1 = n * C, min(T, n * C + C)
                m = t1 - t0
                qc, kc, vc = (_pad_chunk(x, t0, t1, C) for x in (qh_, kh_, vh))
                bc = _pad_chunk(bt, t0, t1, C)
                gc = _pad_chunk(gh, t0, t1, C)
                dOc = _pad_chunk(dO[b, :, h], t0, t1, C)
                # per-pair cumulative decay zeta_i and the transformed tiles
                gam = np.cumsum(gc[:, 0::2], axis=0)
                Th = np.cumsum(gc[:, 1::2], axis=0)
                zeta = np.exp(gam - 1j * Th)                     # [C, dk/2]
                kz, qz = _pairs(kc), _pairs(qc)
                Khz, Kbz, Qhz = zeta * kz, kz / np.conj(zeta), zeta * qz
                Ktz = (np.conj(zeta[-1])[None, :] / np.conj(zeta)) * kz
                Kh, Kb, Qh, Kt = (_unpairs(z) for z in (Khz, Kbz, Qhz, Ktz))
                A = bc[:, None] * np.tril(Kh @ Kb.T, -1)
                IA = np.eye(C) + A
                X = np.linalg.solve(IA, bc[:, None] * np.concatenate([vc, Kh], axis=1))
                Up, W = X[:, :dv], X[:, dv:]
                Mm = np.tril(Qh @ Kb.T)
                S = states[b, h, n]
                U = Up - W @ S.T
                SG = _unpairs(np.conj(zeta[-1])[None, :] * _pairs(S))   # S Gamma_C
                # outputs and state transfer of this chunk
                dU = Mm.T @ dOc + Kt @ dS.T
                dMm = np.tril(dOc @ U.T)
                dQh = dOc @ S + dMm @ Kb
                dKb = dMm.T @ Qh
                dKt = U @ dS
                dW = -dU @ S
                dS_prev = _unpairs(zeta[-1][None, :] * _pairs(dS)) + dOc.T @ Qh - dU.T @ W
                # triangular residual system (I + A) X = R
                Lam = np.linalg.solve(IA.T, np.concatenate([dU, dW], axis=1))
                dA = -np.tril(Lam @ X.T, -1)
                LamU, LamW = Lam[:, :dv], Lam[:, dv:]
                dvc = bc[:, None] * LamU
                dKh = bc[:, None] * LamW
                dbc = np.sum(LamU * vc, axis=1) + np.sum(LamW * Kh, axis=1)
                dbc += np.sum(dA * np.tril(Kh @ Kb.T, -1), axis=1)
                dKh += bc[:, None] * (dA @ Kb)
                dKb += dA.T @ (bc[:, None] * Kh)
                # the per-pair complex factors
                dKhz, dKbz, dQhz, dKtz = (_pairs(x) for x in (dKh, dKb, dQh, dKt))
                dqc = _unpairs(np.conj(zeta) * dQhz)
                dkc = _unpairs(np.conj(zeta) * dKhz + dKbz / zeta
                               + (zeta[-1][None, :] / zeta) * dKtz)
                pKh, pKb = np.conj(dKhz) * Khz, np.conj(dKbz) * Kbz
                pQh, pKt = np.conj(dQhz) * Qhz, np.conj(dKtz) * Ktz
                dgam = (pKh + pQh - pKb - pKt).real
                dTh = (pKh + pQh + pKb + pKt).imag
                pS = np.sum(np.conj(_pairs(dS)) * _pairs(SG), axis=0)    # decay of S
                dgam[-1] += np.sum(pKt, axis=0).real + pS.real
                dTh[-1] += -np.sum(pKt, axis=0).imag - pS.imag
                dgc = np.zeros((C, dk))
                dgc[:, 0::2] = np.cumsum(dgam[::-1], axis=0)[::-1]
                dgc[:, 1::2] = np.cumsum(dTh[::-1], axis=0)[::-1]
                if beta_mode == BETA_KACZMARZ:
                    den = _pad_chunk(norm, t0, t1, C) + eps
                    dkc += (-2.0 * bc * dbc / den)[:, None] * kc
                    dbc = dbc / den
                dq[b, t0:t1, h] = dqc[:m]
                dkk[b, t0:t1, h] = dkc[:m]
                dvv[b, t0:t1, h] = dvc[:m]
                db[b, t0:t1, h] = dbc[:m]
                dg[b, t0:t1, h] = dgc[:m]
                dS = dS_prev
            dS0[b, h] = dS
    return dict(dq=dq, dk=dkk, dv=dvv, dbeta=db, dg=dg, dS0=dS0)
