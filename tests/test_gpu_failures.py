"""Device-side failure reporting (GPU required), without faulting the GPU.

* A bounded wait that runs out: the re-threshold move kernel waits (bounded) for the
  "page read" flag of every earlier page its kept rows move into.  Starting the
  kernel's work counter past page 0 leaves page 0 unclaimed, so its flag is never
  raised; with the wait limit lowered to 20 us, the waits on it give up: the call
  reports SPKV_ERR_TIMEOUT through spkv_cache_check and the rows bound for page 0 are
  not written (page 0 is unchanged).  Every index stays in bounds and every wait ends.
* The debug build (SPKV_DEBUG) checks page-table entries before using them: a page
  number outside the pool, planted on the host, is reported as SPKV_ERR_INDEX by the
  decode attention, which reads nothing outside the pool (its copies of a bad page are
  redirected out of the tensor, where the copy engine fills zeros).
"""
import numpy as np
import pytest
import torch

from sparse_decode_attention_spkv_b200.inputs import workloads as W
from tests import cases as C

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from sparse_decode_attention_spkv_b200 import runner as R
    from sparse_decode_attention_spkv_b200 import spkv as S


def _filled_layer(wl, T0, store_u=True):
    W1, b1, W2, b2 = C.weights(wl)
    p = S.make_params(wl.B, wl.Hq, wl.Hkv, wl.head_dim, wl.d_model, wl.hid, wl.window, wl.tau,
                      S.BF16)
    mp = R.pages_for(T0 + 8)
    layer = R.Layer.create(p, C.dev(W1, "bf16"), C.dev_f32(b1), C.dev_f32(W2), C.dev_f32(b2),
                           num_pages=wl.B * wl.Hkv * mp, max_pages_per_head=mp, store_u=store_u)
    rows = [C.host_rows(wl, 0, b, np.arange(T0 + 1)) for b in range(wl.B)]
    h, q, k, v = (np.stack([r[i] for r in rows]) for i in range(4))
    for c0 in range(0, T0, 512):
        c1 = min(T0, c0 + 512)
        R.prefill_chunk(layer, C.dev(h[:, c0:c1], "bf16"), C.dev(q[:, c0:c1], "bf16"),
                        C.dev(k[:, c0:c1], "bf16"), C.dev(v[:, c0:c1], "bf16"), c0,
                        n_compact=max(0, min(c1, T0 - wl.window) - c0))
    torch.cuda.synchronize()
    return p, layer, (h, q, k, v)


WL = W.small_case("decode32k", cid=64, B=1, Hq=8, Hkv=2, d_model=128, hid=32, ctx=[2000],
                  decode_steps=1, layers=1, keep="fixed25")


def test_rethreshold_wait_gives_up_and_reports_timeout():
    p, layer, _ = _filled_layer(WL, WL.ctx[0])
    c = layer.cache
    n0 = int(c.count[0].item())
    assert n0 > 2 * S.PAGE_ROWS, "head 0 needs rows beyond its first page"
    page0 = int(c.page_table[0, 0].item())
    before = {k: getattr(c, k)[page0].clone() for k in ("K_pool", "V_pool", "pos_pool", "u_pool")}
    # a threshold that keeps about half the rows: rows of head 0's page 1 move into page 0
    u_rows = c.u_pool[c.page_table[0, :(n0 + 63) // 64].long()].flatten()[:n0]
    tau_new = float(u_rows.median().item())
    ws = S.alloc_rethreshold_workspace(p, c)
    ws.view(torch.int32)[0] = 1  # work counter past page 0: page 0 is never claimed
    S.spkv_debug_set_flag_wait_ns(20_000)
    try:
        S.spkv_cache_rethreshold(p, c, layer.ring, tau_new, ws)
        status, flags = S.spkv_cache_check(c)
    finally:
        S.spkv_debug_set_flag_wait_ns(0)
    assert status == S.ERR_TIMEOUT and flags & S.FLAG_TIMEOUT, (status, flags)
    for k, v in before.items():  # nothing was written into the unread page
        assert torch.equal(getattr(c, k)[page0], v), k
    assert int(ws.view(torch.int32)[0].item()) == 0  # the finish kernel reset the counter


def test_debug_build_reports_bad_page_numbers():
    dbg = S.open_library(S.DEBUG_LIB_PATH)
    main = S.lib
    p, layer, (h, q, k, v) = _filled_layer(WL, WL.ctx[0], store_u=False)
    T0 = WL.ctx[0]
    t_pos = torch.full((WL.B,), T0, dtype=torch.int32, device="cuda")
    S.spkv_decode_append(p, layer.cache, layer.ring, t_pos, C.dev(k[:, T0], "bf16"),
                         C.dev(v[:, T0], "bf16"), None, None, 1)
    qt = C.dev(q[:, T0], "bf16")
    o = torch.empty_like(qt)
    S.lib = dbg
    try:
        # a clean state: the checks stay quiet
        S.spkv_decode_attn(p, layer.cache, layer.ring, qt, t_pos, o, None, layer.ws)
        assert S.spkv_cache_check(layer.cache)[0] == S.OK
        # a page number far outside the pool in head 1's table
        layer.cache.page_table[1, 1] = layer.cache.K_pool.shape[0] + 1000
        S.spkv_decode_attn(p, layer.cache, layer.ring, qt, t_pos, o, None, layer.ws)
        status, flags = S.spkv_cache_check(layer.cache)
    finally:
        S.lib = main
    assert status == S.ERR_INDEX and flags & S.FLAG_INDEX, (status, flags)
    assert torch.isfinite(o.float()).all()
