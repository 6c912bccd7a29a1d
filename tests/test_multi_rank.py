"""Multi-rank host logic on CPU with the gloo backend, world size 2: max-over-ranks
timing, job throughput and sharding of independent units (no GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from sparse_decode_attention_spkv_b200 import dist as D


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    w, r, _ = D.init("gloo", timeout_s=60)
    elapsed = [0.25, 0.5][r]                 # rank 1 is slower
    D.barrier(w)
    m = D.max_over_ranks(elapsed, w)
    start, count = D.shard(10, w, r)
    q.put((r, m, D.job_throughput(8 * 20, w, m), start, count))
    D.finalize(w)


def test_two_rank_timing_and_sharding():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [0.5, 0.5]             # both ranks see the slowest time
    assert out[0][2] == pytest.approx(2 * 8 * 20 / 0.5)   # every rank's tokens / max time
    assert [(o[3], o[4]) for o in out] == [(0, 5), (5, 5)]


def test_shard_covers_all_units():
    for n in (1, 7, 64, 257):
        for world in (1, 2, 3, 8):
            spans = [D.shard(n, world, r) for r in range(world)]
            assert sum(c for _, c in spans) == n
            assert spans[0][0] == 0
            for (s0, c0), (s1, _) in zip(spans, spans[1:]):
                assert s0 + c0 == s1
