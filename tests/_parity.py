"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, then compare per tensor with
max relative error = max|gpu - oracle| / max|oracle|."""
import numpy as np
import torch

import oracle
from delta_rule_linear_chunkwise_b200 import binding

GRADS = ("dq", "dk", "dv", "dbeta", "dg", "dS0")


def tol(w):
    """1e-4 for fp32 storage, 2e-2 for bf16 storage with fp32 accumulation."""
    return 1e-4 if w.dtype == "f32" else 2e-2


def rel_err(x, y):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    den = np.max(np.abs(y))
    return float(np.max(np.abs(x - y)) / den) if den > 0 else float(np.max(np.abs(x)))


def run_gpu(w, inp, dST=None, save=True, device="cuda"):
    plan = binding.Plan.for_workload(w, device=device)
    d = {n: (None if x is None else x.to(device)) for n, x in inp.items()}
    dst = None if dST is None else dST.to(device)
    o, ST, saved = plan.fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], save=save)
    gr = plan.bwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], d["dO"], dst,
                  saved if save else None)
    torch.cuda.synchronize()
    assert binding.last_device_error() == binding.DR_OK
    out = dict(o=o, ST=ST, **gr)
    return {n: (None if x is None else x.float().cpu().numpy()) for n, x in out.items()}


def run_oracle(w, inp, heads, dST=None):
    """fp64 oracle on the (b, h) heads listed (all heads if None).

    Returns dict of arrays stacked over the selected heads: o [n, T, dv],
    ST [n, dv, dk], dq/dk [n, T, dk], dv [n, T, dv], dbeta [n, T], dg like g,
    dS0 [n, dv, dk]."""
    B, H = w.B, w.H
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]

    def pick(x, b, h, state=False):
        if x is None:
            return None
        x = x.double().numpy()
        return x[b:b + 1, h:h + 1] if state else x[b:b + 1, :, h:h + 1]

    mode = oracle.BETA_KACZMARZ if w.beta_mode == "kaczmarz" else oracle.BETA_DIRECT
    # Concatenate the selected heads along the batch axis: heads are independent.
    cat = lambda xs: None if xs[0] is None else np.concatenate(xs, axis=0)
    args = {n: cat([pick(inp[n], b, h) for b, h in heads])
            for n in ("q", "k", "v", "beta", "g", "dO")}
    S0 = cat([pick(inp["S0"], b, h, True) for b, h in heads])
    dst = None if dST is None else cat([pick(dST, b, h, True) for b, h in heads])
    gate = oracle.GATE_PHASE if w.gate == "phase" else None
    o, ST = oracle.recurrent_fwd(args["q"], args["k"], args["v"], args["beta"], args["g"],
                                 S0, beta_mode=mode, eps=w.eps, gate=gate)
    gr = oracle.recurrent_bwd(args["q"], args["k"], args["v"], args["beta"], args["g"], S0,
                              args["dO"], dst, beta_mode=mode, eps=w.eps, gate=gate)
    out = dict(o=o[:, :, 0], ST=ST[:, 0], dq=gr["dq"][:, :, 0], dk=gr["dk"][:, :, 0],
               dv=gr["dv"][:, :, 0], dbeta=gr["dbeta"][:, :, 0],
               dg=None if gr["dg"] is None else gr["dg"][:, :, 0], dS0=gr["dS0"][:, 0])
    return out, heads


def select(gpu, heads):
    """Pick the same heads out of full GPU outputs."""
    out = {}
    for n, x in gpu.items():
        if x is None:
            out[n] = None
        elif n in ("ST", "dS0"):
            out[n] = np.stack([x[b, h] for b, h in heads])
        else:
            out[n] = np.stack([x[b, :, h] for b, h in heads])
    return out


def compare(w, gpu, ref, names=("o", "ST") + GRADS):
    errs = {}
    for n in names:
        if ref.get(n) is None:
            assert gpu.get(n) is None or w.gate == "none" or n != "dg"
            continue
        errs[n] = rel_err(gpu[n], ref[n])
    return errs
