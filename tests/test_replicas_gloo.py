"""The multi-GPU run's host logic on CPU: two ranks over the gloo backend
(one process each, as under torchrun) exercising the same helpers bench.py
uses with NCCL on GPUs -- rank seeds, barrier, max-over-ranks timing and the
whole-job throughput."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from quantized_attention_sub_b200 import inputs, replicas
    ws, r, local = replicas.init("gloo", timeout_s=60)
    base = inputs.WORKLOADS["unit"]
    q, _, _ = inputs.generate(inputs.variant(base, seed=replicas.rank_seed(base.seed, r)))
    replicas.barrier(ws)
    # rank r "took" 1.5 * (r + 1) ms for 100 units
    mx = replicas.max_over_ranks(1.5 * (r + 1), ws, "cpu")
    rate = replicas.job_throughput(100.0, mx, ws)
    queue.put((r, ws, local, float(q.float().double().sum()), mx, rate))
    replicas.shutdown(ws)


def test_two_gloo_ranks_time_and_throughput():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(queue.get(timeout=180) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    (r0, w0, l0, s0, m0, t0), (r1, w1, l1, s1, m1, t1) = res
    assert (r0, r1, w0, w1, l0, l1) == (0, 1, 2, 2, 0, 1)
    assert m0 == m1 == 3.0  # the slowest rank's time
    assert t0 == t1 == pytest.approx(100.0 * 2 / 3.0e-3)  # all ranks' units over that time
    assert s0 != s1  # every rank draws its own slices


def test_rank_seeds_are_distinct_and_reproducible():
    from quantized_attention_sub_b200 import inputs, replicas
    base = inputs.WORKLOADS["unit"]
    seeds = [replicas.rank_seed(base.seed, r) for r in range(8)]
    assert len(set(seeds)) == 8 and seeds[0] == base.seed
    a = inputs.generate(inputs.variant(base, seed=seeds[3]))[0]
    b = inputs.generate(inputs.variant(base, seed=seeds[3]))[0]
    assert torch.equal(a, b)


def test_single_rank_needs_no_process_group():
    from quantized_attention_sub_b200 import replicas
    assert replicas.max_over_ranks(2.5, 1) == 2.5
    assert replicas.job_throughput(10.0, 2.0, 1) == pytest.approx(5000.0)
