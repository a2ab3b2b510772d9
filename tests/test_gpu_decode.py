"""Decode parity through the C ABI: the GPU decode step (kernel (a) selection + kernel (b)
reconstruct-and-attend + combine) against the CPU oracle on the SAME stored cache
(oracle-encoded, then stored in the workload precision).

Bar: selected chunk indices bit-exact except ties within 1e-5 of the k-th score
(reported); outputs within max|err| / RMS(out) <= 1e-4 (fp32) or 2e-2 (bf16)."""
import numpy as np
import pytest
import torch

import oracle.lowram_oracle as O
from long_context_decode_02_b200 import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(cuda_device):
    from long_context_decode_02_b200 import lowram
    return lowram


def gpu_decode(L, shape, cache_dev, t, q, variant):
    dev = cache_dev["coef"].device
    cfg = L.make_config(shape, decode_variant=variant)
    ctx = L.Context(cfg, dev.index or 0)
    ws = torch.empty(L.workspace_size(cfg, L.OP_DECODE), dtype=torch.uint8, device=dev)
    k = min(shape.top_k, shape.n_chunks)
    out = torch.empty_like(q)
    sel = torch.full((shape.batch, shape.n_kv_heads, k), -1, dtype=torch.int32, device=dev)
    params = L.layer_params(*(t[n] for n in ("basis", "w1", "b1", "w2", "b2")))
    L.decode_step(ctx, cache_dev, params, q, out, ws, sel_out=sel)
    st = ctx.last_error()
    ctx.close()
    return out, sel, st


def oracle_decode(shape, cache_o, t, q, sel=None):
    p = H.oracle_params(t)
    return O.decode_step(H.f64(q), cache_o, p["basis"], p["w1"], p["b1"], p["w2"], p["b2"],
                         chunk=shape.chunk, top_k=shape.top_k, theta=shape.theta,
                         act=shape.act, sel=sel)


def check_step(L, shape, cache_dev, t_dev, t_cpu, cache_o, q, variant, report):
    out, sel, st = gpu_decode(L, shape, cache_dev, t_dev, q.to(cache_dev["coef"].device), variant)
    assert st == L.OK, L.lowram_status_string(st)
    sel_np = sel.cpu().numpy()
    osel, scores = O.select_chunks(H.f64(q), cache_o["landmark"], shape.top_k)
    ties = H.compare_selection(sel_np, osel, scores, min(shape.top_k, shape.n_chunks))
    report.append(ties)
    # output against the oracle run on the GPU's own selection (identical unless ties)
    want, _ = oracle_decode(shape, cache_o, t_cpu, q, sel=sel_np.astype(np.int64))
    err = H.rel_err(H.f64(out), want)
    assert err <= H.TOL[shape.dtype], (variant, err)
    return err, out


def prepared(shape, layer, device):
    t = H.stored_layer(shape, layer)
    enc = H.oracle_encode(shape, t)
    cache_dev = H.cache_to_device(shape, enc, device)
    cache_o = H.cache_to_oracle(cache_dev)
    t_dev = {k: v.to(device) for k, v in t.items() if k not in ("k", "v")}
    return t, t_dev, cache_dev, cache_o, enc


def test_config0_fp32_two_layers_four_steps(L, cuda_device):
    sh = synth.CONFIGS[0]
    ties = []
    for layer in range(sh.n_layers):
        t, t_dev, cdev, co, _ = prepared(sh, layer, cuda_device)
        for step in range(sh.steps):
            q = synth.queries(sh, layer, step)
            check_step(L, sh, cdev, t_dev, t, co, q, L.DECODE_AUTO, ties)
    H.assert_ties_bounded(sum(ties), sh.n_layers * sh.steps * sh.batch * sh.n_kv_heads,
                          "config0 chunk selection")


@pytest.fixture(scope="module")
def config1_layers(cuda_device):
    sh = synth.CONFIGS[1]
    return sh, [prepared(sh, layer, cuda_device) for layer in range(sh.n_layers)]


@pytest.mark.parametrize("variant", ["tc", "simt"])
def test_config1_bf16(L, config1_layers, variant):
    sh, layers = config1_layers
    v = L.DECODE_TCGEN05 if variant == "tc" else L.DECODE_SIMT
    ties, errs = [], []
    n_steps = 8   # of config 1's 64 steps per layer: each step is a fresh query
    for layer, (t, t_dev, cdev, co, _) in enumerate(layers):
        for step in range(n_steps):
            q = synth.queries(sh, layer, step)
            err, _ = check_step(L, sh, cdev, t_dev, t, co, q, v, ties)
            errs.append(err)
    print(f"config1 {variant}: max rel err {max(errs):.3e}")
    H.assert_ties_bounded(sum(ties), len(layers) * n_steps * sh.batch * sh.n_kv_heads,
                          f"config1 {variant} chunk selection")


def test_config1_tc_and_simt_agree(L, config1_layers):
    sh, layers = config1_layers
    t, t_dev, cdev, co, _ = layers[0]
    q = synth.queries(sh, 0, 5).cuda()
    o1, s1, _ = gpu_decode(L, sh, cdev, t_dev, q, L.DECODE_TCGEN05)
    o2, s2, _ = gpu_decode(L, sh, cdev, t_dev, q, L.DECODE_SIMT)
    assert torch.equal(s1, s2)
    assert H.rel_err(H.f64(o1), H.f64(o2)) <= 2e-2


def test_config1_fp32_rerun(L, cuda_device):
    sh = synth.CONFIGS[1].replace(dtype="f32", n_tokens=8192)
    t, t_dev, cdev, co, _ = prepared(sh, 0, cuda_device)
    ties = []
    for step in range(2):
        check_step(L, sh, cdev, t_dev, t, co, synth.queries(sh, 0, step), L.DECODE_AUTO, ties)


SMALL = synth.CONFIGS[1].replace(name="small", n_tokens=2048, batch=2, seed=77)


@pytest.mark.parametrize("variant", ["tc", "simt"])
@pytest.mark.parametrize("over", [
    dict(top_k=10 ** 6),          # every chunk selected
    dict(top_k=37),               # ragged last tile
    dict(top_k=1),
    dict(res_frac=0.0),           # no residuals
    dict(res_frac=1.0),           # every token a residual
    dict(rank=128, act=synth.ACT_GELU_ERF),
    dict(batch=20, top_k=37),     # 160 (b, h) pairs: more than one per SM
], ids=["all", "ragged", "k1", "nores", "allres", "r128gelu", "manypairs"])
def test_edge_cases(L, cuda_device, variant, over):
    sh = SMALL.replace(**over)
    v = L.DECODE_TCGEN05 if variant == "tc" else L.DECODE_SIMT
    t, t_dev, cdev, co, _ = prepared(sh, 0, cuda_device)
    ties = []
    check_step(L, sh, cdev, t_dev, t, co, synth.queries(sh, 0, 0), v, ties)


@pytest.mark.parametrize("variant", ["tc", "simt"])
def test_exact_ties_go_to_lower_chunk(L, cuda_device, variant):
    sh = SMALL.replace(top_k=20)
    t, t_dev, cdev, co, _ = prepared(sh, 0, cuda_device)
    q = synth.queries(sh, 0, 0)
    # 60 chunks get a copy of each head's best landmark: 61 scores tie exactly at the top
    _, scores = O.select_chunks(H.f64(q), co["landmark"], sh.top_k)
    lm = cdev["landmark"]
    for b in range(sh.batch):
        for h in range(sh.n_kv_heads):
            best = int(np.argmax(scores[b, h]))
            lm[b, h, 100:160] = lm[b, h, best]
    co = H.cache_to_oracle(cdev)
    out, sel, st = gpu_decode(L, sh, cdev, t_dev, q.cuda(),
                              L.DECODE_TCGEN05 if variant == "tc" else L.DECODE_SIMT)
    assert st == L.OK
    osel, _ = O.select_chunks(H.f64(q), co["landmark"], sh.top_k)
    assert np.array_equal(sel.cpu().numpy(), osel)


def test_malformed_cache_is_reported_not_faulted(L, cuda_device):
    sh = SMALL
    t, t_dev, cdev, co, _ = prepared(sh, 0, cuda_device)
    q = synth.queries(sh, 0, 0).cuda()
    for variant in (L.DECODE_TCGEN05, L.DECODE_SIMT):
        bad = {k: v.clone() for k, v in cdev.items()}
        bad["res_idx"].fill_(sh.n_tokens + 5)       # every residual outside its chunk
        _, _, st = gpu_decode(L, sh, bad, t_dev, q, variant)
        assert st == L.ERR_DEVICE_CHECK
        bad = {k: v.clone() for k, v in cdev.items()}
        bad["chunk_ptr"][..., 1:] = sh.n_res + 100  # CSR offsets beyond the residual rows
        _, _, st = gpu_decode(L, sh, bad, t_dev, q, variant)
        assert st == L.ERR_DEVICE_CHECK


def test_full_rank_full_budget_equals_dense_attention(L, cuda_device):
    """r = D, every token a residual, every chunk selected: GPU encode + GPU decode must
    equal exact dense attention over the original keys and values."""
    sh = synth.CONFIGS[0].replace(name="fullrank", n_tokens=512, rank=128, res_frac=1.0,
                                  top_k=10 ** 6, seed=5)
    t = H.stored_layer(sh, 0)
    dev = cuda_device
    cfg = L.make_config(sh)
    ctx = L.Context(cfg)
    cache = L.alloc_cache(cfg, dev)
    td = {k: v.to(dev) for k, v in t.items()}
    params = L.layer_params(*(td[n] for n in ("basis", "w1", "b1", "w2", "b2")))
    ws = torch.empty(L.workspace_size(cfg, L.OP_ENCODE), dtype=torch.uint8, device=dev)
    L.encode(ctx, td["k"], td["v"], params, cache, ws)
    assert ctx.last_error() == L.OK
    q = synth.queries(sh, 0, 0)
    out = torch.empty_like(q, device=dev)
    wsd = torch.empty(L.workspace_size(cfg, L.OP_DECODE), dtype=torch.uint8, device=dev)
    L.decode_step(ctx, cache, params, q.to(dev), out, wsd)
    assert ctx.last_error() == L.OK
    dense = O.dense_attention(H.f64(q), H.f64(t["k"]), H.f64(t["v"]))
    assert H.rel_err(H.f64(out), dense) <= 1e-4
