"""The multi-GPU path of the benchmark (one independent replica per rank, timing reduced by
max over ranks), exercised with two gloo processes on the CPU."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from quantized_decode_attention_kv_b200 import replicas as R
from quantized_decode_attention_kv_b200.workloads import WORKLOADS, make_inputs


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    r, local, w = R.env_ranks()
    R.init("gloo", w, timeout_s=60)
    times = [0.25, 0.75]
    job = R.max_over_ranks(times[r], w)
    rate = R.job_throughput(100.0, w, job)
    wl = WORKLOADS["gpt2_prod_2bit"]
    K, V, q = make_inputs(wl, B=1, T=4, Hkv=1, Hq=1, layer=R.replica_layer(r))
    R.barrier(w)
    out.put((r, job, rate, float(K.float().sum()), float(q.float().sum())))
    R.finish(w)


def test_two_gloo_ranks_share_the_max_time_and_use_distinct_inputs():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, job0, rate0, k0, q0), (r1, job1, rate1, k1, q1) = res
    assert job0 == job1 == 0.75          # every rank sees the slowest rank's time
    assert rate0 == rate1 == pytest.approx(2 * 100.0 / 0.75)
    assert k0 != k1 and q0 != q1         # each replica replays its own layer


def test_single_rank_needs_no_process_group():
    assert R.max_over_ranks(1.5, 1) == 1.5
    assert R.job_throughput(10.0, 1, 2.0) == 5.0
    # the same layer always gives the same inputs
    wl = WORKLOADS["tiny_single_head_fp32"]
    a = make_inputs(wl, T=8, layer=3)[0]
    b = make_inputs(wl, T=8, layer=3)[0]
    assert torch.equal(a, b)
