"""Decode over the compressed prefix plus an uncompressed suffix of generated tokens
(lowram_decode_step_suffix), through the C ABI, against the oracle's
decode_step_with_suffix: one softmax over the selected chunks' rebuilt tokens and every
suffix token (long generation keeps recent tokens uncompressed; agihunt summary,
limitations paragraph). Bars as in the decode tests: selections bit-exact except ties,
outputs within the bf16 tolerance."""
import numpy as np
import pytest
import torch

import oracle.lowram_oracle as O
from long_context_decode_02_b200 import synth
from tests import helpers as H
from tests.test_gpu_decode import prepared

pytestmark = pytest.mark.gpu

SMALL = synth.CONFIGS[1].replace(name="suffix", n_tokens=2048, batch=2, seed=81)
S_MAX = 1100


@pytest.fixture(scope="module")
def L(cuda_device):
    from long_context_decode_02_b200 import lowram
    return lowram


@pytest.fixture(scope="module")
def suffix_kv():
    g = torch.Generator().manual_seed(82)
    shape = (SMALL.batch, S_MAX, SMALL.n_kv_heads, SMALL.head_dim)
    ks = torch.randn(shape, generator=g).to(torch.bfloat16).contiguous()
    vs = torch.randn(shape, generator=g).to(torch.bfloat16).contiguous()
    return ks, vs


@pytest.mark.parametrize("variant", ["tc", "simt"])
@pytest.mark.parametrize("n_suffix", [0, 1, 100, 1040])
def test_suffix_decode_matches_oracle(L, cuda_device, suffix_kv, variant, n_suffix):
    sh = SMALL
    dev = cuda_device
    t, t_dev, cdev, co, _ = prepared(sh, 0, dev)
    ks, vs = suffix_kv
    v = L.DECODE_TCGEN05 if variant == "tc" else L.DECODE_SIMT
    cfg = L.make_config(sh, decode_variant=v)
    ctx = L.Context(cfg, dev.index or 0)
    ws = torch.empty(L.suffix_workspace_size(cfg, S_MAX), dtype=torch.uint8, device=dev)
    params = L.layer_params(*(t_dev[n] for n in ("basis", "w1", "b1", "w2", "b2")))
    p = H.oracle_params(t)
    k = min(sh.top_k, sh.n_chunks)
    q = synth.queries(sh, 0, n_suffix % 7)
    out = torch.empty_like(q, device=dev)
    sel = torch.empty(sh.batch, sh.n_kv_heads, k, dtype=torch.int32, device=dev)
    L.decode_step_suffix(ctx, cdev, params, q.to(dev), ks.to(dev), vs.to(dev), n_suffix, out,
                         ws, sel_out=sel)
    assert ctx.last_error() == L.OK
    ctx.close()
    sel_np = sel.cpu().numpy()
    osel, scores = O.select_chunks(H.f64(q), co["landmark"], sh.top_k)
    ties = H.compare_selection(sel_np, osel, scores, k)
    H.assert_ties_bounded(ties, sh.batch * sh.n_kv_heads, "suffix decode selection")
    want, _ = O.decode_step_with_suffix(H.f64(q), co, p["basis"], p["w1"], p["b1"], p["w2"],
                                        p["b2"], H.f64(ks[:, :n_suffix]), H.f64(vs[:, :n_suffix]),
                                        chunk=sh.chunk, top_k=sh.top_k, theta=sh.theta,
                                        act=sh.act, sel=sel_np.astype(np.int64))
    err = H.rel_err(H.f64(out), want)
    print(f"suffix decode {variant} n={n_suffix}: rel err {err:.2e}")
    assert err <= H.TOL["bf16"]


def test_suffix_full_rank_equals_dense_over_prefix_and_suffix(L, cuda_device, suffix_kv):
    """Full rank, every token a residual, every chunk selected: GPU encode, then decode
    with a suffix, equals dense attention over the prefix and suffix together."""
    sh = SMALL.replace(name="suffix-fullrank", n_kv_heads=1, n_q_heads=4, rank=128,
                       res_frac=1.0, top_k=10 ** 6, n_tokens=1024, seed=83)
    dev = cuda_device
    t = H.stored_layer(sh, 0)
    td = {k: v.to(dev) for k, v in t.items()}
    cfg = L.make_config(sh)
    ctx = L.Context(cfg, dev.index or 0)
    cache = L.alloc_cache(cfg, dev)
    params = L.layer_params(*(td[n] for n in ("basis", "w1", "b1", "w2", "b2")))
    wse = torch.empty(L.workspace_size(cfg, L.OP_ENCODE), dtype=torch.uint8, device=dev)
    L.encode(ctx, td["k"], td["v"], params, cache, wse)
    ks, vs = (x[:, :, :1].contiguous() for x in suffix_kv)
    n = 700
    ws = torch.empty(L.suffix_workspace_size(cfg, ks.shape[1]), dtype=torch.uint8, device=dev)
    q = synth.queries(sh, 0, 0)
    out = torch.empty_like(q, device=dev)
    L.decode_step_suffix(ctx, cache, params, q.to(dev), ks.to(dev), vs.to(dev), n, out, ws)
    assert ctx.last_error() == L.OK
    ctx.close()
    dense = O.dense_attention(H.f64(q), np.concatenate([H.f64(t["k"]), H.f64(ks[:, :n])], 1),
                              np.concatenate([H.f64(t["v"]), H.f64(vs[:, :n])], 1))
    assert H.rel_err(H.f64(out), dense) <= 2e-2
