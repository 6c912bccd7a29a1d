"""Run one kernel of the SP-KV path on a small, fixed configuration (for profilers).

    python -m sparse_decode_attention_spkv_b200.kernel_driver decode  [--layers 1] [--steps 3]
                                      [--decode-step attn-first|one-stream|split|fused]
                                      [--workload decode32k|ragged128k]
    python -m sparse_decode_attention_spkv_b200.kernel_driver score   [--tokens 8]
    python -m sparse_decode_attention_spkv_b200.kernel_driver compact [--rows 4096] [--source chunk|ring]
    python -m sparse_decode_attention_spkv_b200.kernel_driver prefill [--chunk 4096]
    python -m sparse_decode_attention_spkv_b200.kernel_driver rethreshold [--steps 2]
    python -m sparse_decode_attention_spkv_b200.kernel_driver soft [--seq 8192]

``decode`` builds the decode32k state (batch 8, 32K context, ~300 MB of live K/V per
layer, more than L2; or the ragged128k state, batch 4, contexts 128K..32K) for a few
layers and runs eager decode steps (one-stream: attention first, then the fused score
and update on the same stream); the others run
their kernel a few times on decode32k / prefill16k shapes.  Prints nothing but a
completion line: timings come from the profiler.
"""
from __future__ import annotations

import argparse

import torch

from . import runner as R
from . import spkv as S
from .inputs import device as D
from .inputs import gen
from .inputs import workloads as W


def _layer(wl, rows_per_head, device="cuda"):
    p = S.make_params(wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau,
                      S.BF16)
    W1 = torch.from_numpy(wl.w1(0)).to(torch.bfloat16).to(device)
    b1 = torch.from_numpy(wl.b1(0)).to(device)
    W2 = torch.from_numpy(wl.w2(0)).to(device)
    b2 = torch.from_numpy(wl.b2(0)).to(device)
    mp = R.pages_for(rows_per_head)
    return R.Layer.create(p, W1, b1, W2, b2, wl.B * wl.Hkv * mp, mp, device)


def run_decode(args):
    from .states import DecodeStep, build_decode_state
    wl = W.WORKLOADS[args.workload]
    p, Ls, inp = build_decode_state(wl, args.layers, args.steps, torch.device("cuda"))
    step = DecodeStep(p, Ls, "cuda", split=args.decode_step in ("attn-first", "split"),
                      attn_first=args.decode_step in ("attn-first", "one-stream"))
    for i in range(args.steps):
        step.launch(inp["h"][i], inp["q"][i], inp["k"][i], inp["v"][i], inp["t"][i])
    torch.cuda.synchronize()


def run_score(args):
    wl = W.WORKLOADS["decode32k"]
    L = _layer(wl, 64)
    h = torch.empty((args.tokens, wl.d_model), dtype=torch.bfloat16, device="cuda")
    D.fill_normal(h, wl.key(0, gen.T_H), 1.0)
    for _ in range(args.steps):
        R.score(L, h, args.tokens)
    torch.cuda.synchronize()


def run_compact(args):
    """--source chunk: one prefill16k chunk (batch 1, args.rows tokens, 8 key heads)
    compacted from the chunk tensors, args.steps times (consecutive chunks);
    --source ring: one serving bulk pass (batch 32, the 128 buffered tokens of every row,
    8 key heads) compacted from the ring, args.steps times."""
    if args.source == "ring":
        wl = W.WORKLOADS["serving"]
        n = wl.bulk
        L = _layer(wl, (args.steps + 1) * n)
        D.fill_normal(L.ring.K_win, wl.key(0, gen.T_K), wl.qkv_scale)
        D.fill_normal(L.ring.V_win, wl.key(0, gen.T_V), wl.qkv_scale)
        h = torch.empty((wl.B * n, wl.d_model), dtype=torch.bfloat16, device="cuda")
        D.fill_normal(h, wl.key(0, gen.T_H), 1.0)
        u, z = R.score(L, h, wl.B * n)
        for i in range(args.steps):
            src = torch.full((wl.B,), i * n, dtype=torch.int32, device="cuda")
            S.spkv_write_compact(L.p, L.cache, L.ring, S.SRC_RING, None, None, z, u, src, n, n)
        torch.cuda.synchronize()
        return
    wl = W.WORKLOADS["prefill16k"]
    n = args.rows
    L = _layer(wl, 4 * n)
    k = torch.empty((1, n, wl.Hkv, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    h = torch.empty((n, wl.d_model), dtype=torch.bfloat16, device="cuda")
    D.fill_normal(k, wl.key(0, gen.T_K), wl.qkv_scale)
    D.fill_normal(v, wl.key(0, gen.T_V), wl.qkv_scale)
    D.fill_normal(h, wl.key(0, gen.T_H), 1.0)
    u, z = R.score(L, h, n)
    for i in range(args.steps):
        src = torch.full((1,), i * n, dtype=torch.int32, device="cuda")
        S.spkv_write_compact(L.p, L.cache, L.ring, S.SRC_CHUNK, k, v, z, u, src, n, n)
    torch.cuda.synchronize()


def run_prefill(args):
    wl = W.WORKLOADS["prefill16k"]
    T = wl.ctx[0]
    c = args.chunk
    L = _layer(wl, T)
    Tt = wl.T_total
    for c0 in range(0, min(T, c * args.steps), c):
        h = torch.empty((1, c, wl.d_model), dtype=torch.bfloat16, device="cuda")
        q = torch.empty((1, c, wl.Hq, wl.head_dim), dtype=torch.bfloat16, device="cuda")
        k = torch.empty((1, c, wl.Hkv, wl.head_dim), dtype=torch.bfloat16, device="cuda")
        v = torch.empty_like(k)
        D.fill_normal(h, wl.key(0, gen.T_H), 1.0, offset=c0 * wl.d_model)
        D.fill_rope(q, wl.key(0, gen.T_Q), c0, Tt, wl.qkv_scale, wl.rope_base)
        D.fill_rope(k, wl.key(0, gen.T_K), c0, Tt, wl.qkv_scale, wl.rope_base)
        D.fill_normal(v, wl.key(0, gen.T_V), wl.qkv_scale, offset=c0 * wl.Hkv * wl.head_dim)
        R.prefill_chunk(L, h, q, k, v, c0)
    torch.cuda.synchronize()


def run_rethreshold(args):
    """One decode32k layer with utilities kept, re-thresholded at the median stored
    utility; the cache is restored from a copy before each repetition."""
    from .states import build_decode_state
    wl = W.small_case("decode32k", layers=1)
    p, Ls, _ = build_decode_state(wl, 1, 1, torch.device("cuda"), store_u=True)
    c = Ls[0].cache
    saved = {k: getattr(c, k).clone() for k in ("K_pool", "V_pool", "pos_pool", "u_pool", "count",
                                                  "count_prev", "page_table")}
    ws = S.alloc_rethreshold_workspace(p, c)
    n = int(c.count.sum().item())
    tau = float(c.u_pool.flatten()[: max(1, n)].median().item())
    for _ in range(args.steps):
        for k, v in saved.items():
            getattr(c, k).copy_(v)
        S.spkv_cache_rethreshold(p, c, Ls[0].ring, tau, ws)
    torch.cuda.synchronize()


def run_soft(args):
    """Soft-gated attention over one sequence with the prefill16k shapes."""
    wl = W.WORKLOADS["prefill16k"]
    T = args.seq
    bf = torch.bfloat16
    p = S.make_params(1, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau, S.BF16)
    q = torch.empty((1, T, wl.Hq, wl.head_dim), dtype=bf, device="cuda")
    k = torch.empty((1, T, wl.Hkv, wl.head_dim), dtype=bf, device="cuda")
    v = torch.empty_like(k)
    D.fill_rope(q, wl.key(0, gen.T_Q), 0, wl.T_total, wl.qkv_scale, wl.rope_base)
    D.fill_rope(k, wl.key(0, gen.T_K), 0, wl.T_total, wl.qkv_scale, wl.rope_base)
    D.fill_normal(v, wl.key(0, gen.T_V), wl.qkv_scale)
    u = torch.rand((1, T, wl.Hkv), device="cuda") * 0.6 + 0.2
    o = torch.empty_like(q)
    ws = torch.empty(S.spkv_soft_attn_workspace_bytes(p, T), dtype=torch.uint8, device="cuda")
    for _ in range(args.steps):
        S.spkv_soft_attn(p, q, k, v, u, T, 0.01, 1e6, o, None, ws)
    torch.cuda.synchronize()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel", choices=["decode", "score", "compact", "prefill", "rethreshold", "soft"])
    ap.add_argument("--layers", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--tokens", type=int, default=8)
    ap.add_argument("--rows", type=int, default=4096)
    ap.add_argument("--chunk", type=int, default=4096)
    ap.add_argument("--seq", type=int, default=8192)
    ap.add_argument("--source", default="chunk", choices=["chunk", "ring"])
    ap.add_argument("--decode-step", default="attn-first",
                    choices=["attn-first", "one-stream", "split", "fused"])
    ap.add_argument("--workload", default="decode32k", choices=["decode32k", "ragged128k"])
    args = ap.parse_args()
    torch.cuda.set_device(0)
    {"decode": run_decode, "score": run_score, "compact": run_compact, "prefill": run_prefill,
     "rethreshold": run_rethreshold, "soft": run_soft}[args.kernel](args)
    st, flags = (S.OK, 0)
    print(f"kernel_driver {args.kernel} done")


if __name__ == "__main__":
    main()
