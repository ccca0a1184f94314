"""Host-side logic of bench.py, on the CPU: the algorithmic work model and the
multi-rank aggregation (max over ranks of the timed region; whole-job
throughput), the latter exercised with two gloo ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
from delta_rule_linear_chunkwise_b200 import WORKLOADS


def test_algorithmic_model_matches_per_token_head_figures():
    w = WORKLOADS["kda_bf16_b4h16t8192"]
    flops, nbytes = bench.algorithmic_step(w)
    th = w.token_heads
    assert flops == th * 638_976           # 38 C d + 20 d^2 at C = 64, d = 128
    state = w.B * w.H * 128 * 128 * 4 * 2  # S_T written, dS0 written
    assert nbytes == th * 4364 + state     # KDA: per-channel g and dg in fp32
    g = WORKLOADS["gdn_bf16_b8h16t4096"]
    _, gbytes = bench.algorithmic_step(g)
    assert gbytes == g.token_heads * 2840 + g.B * g.H * 128 * 128 * 4 * 2


def test_phase_gate_step_model():
    # SFDA workload: the same fwd+bwd model as KDA (the pair gate has d_k fp32
    # values per token, like the per-channel gate, and so does its gradient)
    w = WORKLOADS["sfda_bf16_b4h16t8192"]
    kda = WORKLOADS["kda_bf16_b4h16t8192"]
    assert bench.algorithmic_step(w) == bench.algorithmic_step(kda)
    flops, nbytes = bench.algorithmic_step(w)
    th, C, d = w.token_heads, w.chunk, w.dk
    assert flops == th * (38 * C * d + 20 * d * d)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        m = bench.reduce_max(mine, "cpu")
        v = bench.aggregate_tokens_per_s(world, 32768, 4, m)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_whole_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in got:
        assert m == 15.0
        assert v == pytest.approx(2 * 32768 * 4 / 0.015)


def test_single_process_reduce_is_identity():
    assert bench.reduce_max(3.5, "cpu") == 3.5
