"""Chunkwise gated delta-rule linear attention on B200 (sm_100a).

The operator is the chunkwise (WY / UT-transform) forward and the
triangular-residual (ReWY) backward of

    S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t

for DeltaNet (no gate), GDN (scalar gate), KDA (per-channel gate) and KLA
(beta_t = eta_t / (||k_t||^2 + eps)).  All arithmetic runs in hand-written
CUDA kernels behind the C ABI declared in ``include/dr.h``; this package is the
thin ctypes binding to that library.
"""
from .workloads import HEADLINE, WORKLOADS, Workload, make_inputs  # noqa: F401
