"""Disjoint batch shards (GPU required): the state and decode step of a batch built as
two shards, each drawing its rows by global row index, equal the state and step of the
whole batch row for row (what N ranks of the benchmark serve together)."""
import numpy as np
import pytest
import torch

from sparse_decode_attention_spkv_b200.inputs import workloads as W
from tests import cases as C

pytestmark = pytest.mark.gpu


def test_two_shards_equal_the_whole_batch():
    from sparse_decode_attention_spkv_b200 import runner as R
    from sparse_decode_attention_spkv_b200.states import build_decode_state
    dev = torch.device("cuda")
    whole = W.small_case("decode32k", cid=80, B=4, d_model=256, hid=64, ctx=[1500] * 4,
                         decode_steps=2, layers=1)
    half = W.small_case("decode32k", cid=80, B=2, d_model=256, hid=64, ctx=[1500] * 2,
                        decode_steps=2, layers=1)
    # the same T_total for both (the generator's row stride), as in the benchmark
    assert whole.T_total == half.T_total
    outs = {}
    for name, wl, row0 in (("whole", whole, 0), ("lo", half, 0), ("hi", half, 2)):
        p, (L,), inp = build_decode_state(wl, 1, 2, dev, row0=row0)
        res = []
        for i in range(2):
            o, _, z = R.decode_step(L, inp["t"][i], inp["h"][i][0], inp["q"][i][0],
                                    inp["k"][i][0], inp["v"][i][0])
            res.append((o.float().cpu(), z.cpu()))
        outs[name] = (res, R.cache_lists(L))
    for i in range(2):
        o_w, z_w = outs["whole"][0][i]
        o_s = torch.cat([outs["lo"][0][i][0], outs["hi"][0][i][0]])
        z_s = torch.cat([outs["lo"][0][i][1], outs["hi"][0][i][1]])
        assert torch.equal(z_w, z_s), f"step {i}: gates"
        # the split-K chunking depends on the batch, so the sums may differ in rounding
        C.check_attn(o_s.numpy(), o_w.numpy(), "bf16", f"step {i}: shards vs whole batch")
    lists_w = outs["whole"][1]
    lists_s = outs["lo"][1] + outs["hi"][1]
    assert len(lists_w) == len(lists_s)
    assert all(np.array_equal(a, b) for a, b in zip(lists_w, lists_s)), "cache lists"
