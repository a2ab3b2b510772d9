"""Periodic re-compression of the generated suffix on the GPU (lowram_append), against
the oracle's encode_block and append_block: a block of whole chunks of generated tokens
is compressed under its own context at its true positions (chunk_pos), then appended
after the compressed prefix; decode runs over the result.

The pages name the periodic compression of the generated suffix (agihunt summary,
limitations paragraph); the reading (the block's own residual budget, the prefix left as
it is) is the oracle's.

Bars: the appended arrays equal the two GPU caches concatenated, bit for bit (token
indices moved by the prefix's tokens, CSR offsets by its rows, the larger norm bound);
the block's encode matches the oracle's encode_block (coefficients within one storage
rounding, residual picks bit-exact except near-ties, reported and bounded); decode over
the appended cache selects like the oracle (near-ties bounded) and its output is within
the bf16 tolerance; a result without chunk positions refuses a block that is not
contiguous after the prefix (LOWRAM_ERR_DEVICE_CHECK)."""
import numpy as np
import pytest
import torch

import oracle.lowram_oracle as O
from long_context_decode_02_b200 import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu

SHAPE = synth.CONFIGS[1].replace(name="append-small", n_tokens=4096 + 512, batch=2, seed=71)
T0 = 4096


@pytest.fixture(scope="module")
def L(cuda_device):
    from long_context_decode_02_b200 import lowram
    return lowram


def encode_part(L, sh, td, params, dev, t0, t1, cfg):
    ctx = L.Context(cfg, dev.index or 0)
    cache = L.alloc_cache(cfg, dev)
    if cfg.n_positions > cfg.n_tokens:   # the block: its chunks' true positions
        nc = cfg.n_tokens // sh.chunk
        cache["chunk_pos"].copy_(torch.arange(t0 // sh.chunk, t0 // sh.chunk + nc,
                                              dtype=torch.int32, device=dev).expand(sh.batch, nc))
    ws = torch.empty(L.workspace_size(cfg, L.OP_ENCODE), dtype=torch.uint8, device=dev)
    L.encode(ctx, td["k"][:, t0:t1].contiguous(), td["v"][:, t0:t1].contiguous(), params,
             cache, ws)
    torch.cuda.synchronize()
    assert ctx.last_error() == L.OK
    return ctx, cache


@pytest.fixture(scope="module")
def appended(L, cuda_device):
    sh, dev = SHAPE, cuda_device
    T = sh.n_tokens
    nres_p, nres_b = int(sh.res_frac * T0), int(sh.res_frac * (T - T0))
    t = H.stored_layer(sh, 0)
    td = {k: v.to(dev) for k, v in t.items()}
    params = L.layer_params(*(td[n] for n in ("basis", "w1", "b1", "w2", "b2")))
    cfg_p = L.make_config(sh, n_tokens=T0, n_res=nres_p, n_positions=0)
    cfg_b = L.make_config(sh, n_tokens=T - T0, n_res=nres_b, n_positions=T)
    cfg_d = L.make_config(sh, n_tokens=T, n_res=nres_p + nres_b, n_positions=0)
    ctx_p, pre = encode_part(L, sh, td, params, dev, 0, T0, cfg_p)
    ctx_b, blk = encode_part(L, sh, td, params, dev, T0, T, cfg_b)
    ctx_d = L.Context(cfg_d, dev.index or 0)
    dst = L.alloc_cache(cfg_d, dev)
    L.append(ctx_d, dst, ctx_p, pre, ctx_b, blk)
    torch.cuda.synchronize()
    assert ctx_d.last_error() == L.OK
    return dict(sh=sh, t=t, td=td, params=params, pre=pre, blk=blk, dst=dst, ctx=ctx_d,
                cfg=cfg_d, nres=(nres_p, nres_b), ctxs=(ctx_p, ctx_b))


def test_append_concatenates(L, appended):
    a = appended
    pre, blk, dst = a["pre"], a["blk"], a["dst"]
    for name, dim in (("coef", 1), ("landmark", 2), ("res_val", 2)):
        want = torch.cat([pre[name], blk[name]], dim=dim)
        assert torch.equal(dst[name], want), name
    assert torch.equal(dst["res_idx"], torch.cat([pre["res_idx"], blk["res_idx"] + T0], dim=2))
    n_p = pre["chunk_ptr"].shape[2] - 1
    assert torch.equal(dst["chunk_ptr"],
                       torch.cat([pre["chunk_ptr"][:, :, :n_p], blk["chunk_ptr"] + a["nres"][0]],
                                 dim=2))
    assert torch.equal(dst["landmark_norm"], torch.maximum(pre["landmark_norm"],
                                                           blk["landmark_norm"]))


def test_block_encode_matches_oracle(L, appended):
    a = appended
    sh, t = a["sh"], a["t"]
    p = H.oracle_params(t)
    want = O.encode_block(H.f64(t["k"][:, T0:]), H.f64(t["v"][:, T0:]), p["basis"], p["w1"],
                          p["b1"], p["w2"], p["b2"], chunk=sh.chunk, n_res=a["nres"][1],
                          theta=sh.theta, act=sh.act, store=H.STORE[sh.dtype],
                          first_position=T0)
    got = a["blk"]
    # coefficients: the GPU's fp32 value rounds to the same bf16 value, or to a neighbour
    # when the exact value lies within fp32 error of a rounding midpoint
    gc, wc = H.f64(got["coef"]), want["coef"]
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(wc), 1e-30))) - 7)
    assert np.all(np.abs(gc - wc) <= ulp * 1.01 + 1e-6 * np.abs(wc).max())
    # the block's residual picks: its own largest errors, near-ties reported and bounded
    got_idx = got["res_idx"].cpu().numpy()
    ties = H.compare_selection(got_idx, want["res_idx"], want["err"], a["nres"][1])
    H.assert_ties_bounded(ties, sh.batch * sh.n_kv_heads, "block residual pick")


def test_decode_over_appended_cache(L, appended, cuda_device):
    a = appended
    sh, dev = a["sh"], cuda_device
    cfg = a["cfg"]
    ctx = a["ctx"]
    ws = torch.empty(L.workspace_size(cfg, L.OP_DECODE), dtype=torch.uint8, device=dev)
    p = H.oracle_params(a["t"])
    co = H.cache_to_oracle(a["dst"])
    for step in range(2):
        q = synth.queries(sh, 0, step).to(dev)
        out = torch.empty_like(q)
        sel = torch.empty(sh.batch, sh.n_kv_heads, sh.top_k, dtype=torch.int32, device=dev)
        L.decode_step(ctx, a["dst"], a["params"], q, out, ws, sel_out=sel)
        torch.cuda.synchronize()
        assert ctx.last_error() == L.OK
        qn = H.f64(q)
        osel, scores = O.select_chunks(qn, co["landmark"], sh.top_k)
        g = sel.cpu().numpy()
        ties = H.compare_selection(g, osel, scores, sh.top_k)
        H.assert_ties_bounded(ties, sh.batch * sh.n_kv_heads, "appended-cache selection")
        want, _ = O.decode_step(qn, co, p["basis"], p["w1"], p["b1"], p["w2"], p["b2"],
                                chunk=sh.chunk, top_k=sh.top_k, theta=sh.theta, act=sh.act,
                                sel=g.astype(np.int64))
        assert H.rel_err(H.f64(out), want) <= H.TOL[sh.dtype]


def test_append_keeps_positions_and_checks_contiguity(L, appended, cuda_device):
    """A result with chunk positions gets 0 .. N_p-1 then the block's; one without them
    refuses a block whose positions do not follow the prefix."""
    a = appended
    sh, dev = a["sh"], cuda_device
    T = sh.n_tokens
    ctx_p, ctx_b = a["ctxs"]
    cfg_e = L.make_config(sh, n_tokens=T, n_res=sum(a["nres"]), n_positions=T + 8 * sh.chunk)
    ctx_e = L.Context(cfg_e, dev.index or 0)
    dst = L.alloc_cache(cfg_e, dev)
    L.append(ctx_e, dst, ctx_p, a["pre"], ctx_b, a["blk"])
    torch.cuda.synchronize()
    assert ctx_e.last_error() == L.OK
    n_p, n_b = T0 // sh.chunk, (T - T0) // sh.chunk
    want = torch.arange(n_p + n_b, dtype=torch.int32, device=dev).expand(sh.batch, -1)
    assert torch.equal(dst["chunk_pos"], want)
    # shift the block's positions by one chunk: no longer contiguous after the prefix
    blk = dict(a["blk"])
    blk["chunk_pos"] = (a["blk"]["chunk_pos"] + 1).contiguous()
    dst2 = L.alloc_cache(a["cfg"], dev)
    ctx2 = L.Context(a["cfg"], dev.index or 0)
    L.append(ctx2, dst2, ctx_p, a["pre"], ctx_b, blk)
    torch.cuda.synchronize()
    assert ctx2.last_error() == L.ERR_DEVICE_CHECK
    # mismatched sizes are refused on the host
    with pytest.raises(L.LowRAMError):
        L.append(ctx_e, dst, ctx_b, a["blk"], ctx_p, a["pre"])
