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


def _split_worker(rank, world, port, q):
    """Rank r holds slice r of a sequence's keys: it computes its partial attention over
    that slice alone (the oracle's Eq. (3) on the slice), the ranks all-gather their
    partials with the library's exchange helper, and every rank merges them (the
    oracle's log-sum-exp merge): each must recover the attention over the whole key set."""
    import numpy as np
    import torch
    from oracle import spkv_oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    w, r, _ = D.init("gloo", timeout_s=60)
    rng = np.random.default_rng(5)                      # the same problem on every rank
    B, Hq, Hkv, d, T, win = 2, 4, 2, 16, 300, 32
    G = Hq // Hkv
    Q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, T, Hkv, d))
    V = rng.standard_normal((B, T, Hkv, d))
    z = (rng.random((B, T, Hkv)) < 0.3).astype(np.uint8)
    t = T - 1
    lo, hi = [(0, 150), (150, T)][r]                     # rank r's slice of the positions
    o_part = np.zeros((B, Hq, d))
    lse_part = np.full((B, Hq), -np.inf)
    s = np.arange(T)
    for b in range(B):
        for kh in range(Hkv):
            mask = O.visible(t, s, z[b, :, kh], win) & (s >= lo) & (s < hi)
            if not mask.any():
                continue
            for g in range(G):
                o_part[b, kh * G + g], lse_part[b, kh * G + g] = O.attend(
                    Q[b, kh * G + g], K[b, :, kh], V[b, :, kh], mask)
    o_all = torch.empty((w, B, Hq, d), dtype=torch.float32)
    lse_all = torch.empty((w, B, Hq), dtype=torch.float32)
    D.all_gather_partials(torch.tensor(o_part, dtype=torch.float32),
                          torch.tensor(lse_part, dtype=torch.float32), o_all, lse_all)
    o_m, lse_m = O.merge(o_all.double().numpy(), lse_all.double().numpy())
    err = 0.0
    for b in range(B):
        o_ref, lse_ref = O.gated_attention(Q[b][None], K[b], V[b], z[b], win, [t])
        err = max(err, float(np.max(np.abs(o_m[b] - o_ref[0]))),
                  float(np.max(np.abs(lse_m[b] - lse_ref[0]))))
    mine = float(np.max(np.abs(o_all[r].double().numpy() - o_part)))  # own slot = own partial
    q.put((r, err, mine))
    D.finalize(w)


def test_two_rank_sequence_split_exchange():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, err, mine in out:
        assert mine < 1e-6, f"rank {r}: its own partial is not in its slot"
        assert err < 1e-5, f"rank {r}: merged partials differ from the whole-set attention ({err})"


def _rows_worker(rank, world, port, q):
    """Disjoint batch shards: rank r serves global rows shard(B, world, r) and draws their
    inputs by global row index; the ranks' decode outputs (the oracle's, on the drawn
    inputs), gathered, equal the single-process outputs row for row."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from oracle import spkv_oracle as O
    from sparse_decode_attention_spkv_b200.inputs import workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    w, r, _ = D.init("gloo", timeout_s=60)
    wl = W.small_case("tiny", B=4, ctx=[200] * 4, decode_steps=1)
    row0, n = D.shard(wl.B, w, r)
    T = wl.ctx[0] + 1
    z = np.zeros((T, wl.Hkv), dtype=np.uint8)
    z[::3] = 1
    outs = []
    for b in range(row0, row0 + n):                     # global row indices
        pos = np.arange(T)
        o, _ = O.gated_attention(wl.q_rows(0, b, [T - 1]), wl.k_rows(0, b, pos),
                                 wl.v_rows(0, b, pos), z, wl.window, [T - 1])
        outs.append(o[0])
    mine = torch.tensor(np.stack(outs))
    got = [torch.empty_like(mine) for _ in range(w)]
    dist.all_gather(got, mine)
    q.put((r, torch.cat(got).numpy()))
    D.finalize(w)


def test_two_rank_disjoint_batch_rows():
    import numpy as np
    from oracle import spkv_oracle as O
    from sparse_decode_attention_spkv_b200.inputs import workloads as W
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rows_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=120) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = W.small_case("tiny", B=4, ctx=[200] * 4, decode_steps=1)
    T = wl.ctx[0] + 1
    z = np.zeros((T, wl.Hkv), dtype=np.uint8)
    z[::3] = 1
    want = np.stack([O.gated_attention(wl.q_rows(0, b, [T - 1]), wl.k_rows(0, b, np.arange(T)),
                                       wl.v_rows(0, b, np.arange(T)), z, wl.window, [T - 1])[0][0]
                     for b in range(wl.B)])
    for r, got in out:
        assert got.shape == want.shape
        assert np.max(np.abs(got - want)) < 1e-6, f"rank {r}: gathered rows differ"
