"""Full-size parity, in the launch configuration the bench times, at two shapes: the
headline Llama-3-8B-shaped layer (batch 8, 128K context, rank 160, top-256 chunks, 20%
residuals, bf16) and the Mistral-7B-shaped long-context layer (batch 4, 262144 tokens,
RoPE theta 1e6, rank 128, 15% residuals), whose RoPE angles reach position 262143. The
oracle checks sampled (batch, KV head) pairs one by one, and properties that hold at any
size check the rest."""
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


@pytest.fixture(scope="module", params=[2, 3], ids=["llama8b-b8-128k", "mistral7b-b4-262k"])
def full_layer(L, cuda_device, request):
    sh = synth.CONFIGS[request.param]
    dev = cuda_device
    basis = synth.group_basis(sh, 0)
    w = synth.layer_weights(sh, 0)
    st = sh.torch_dtype
    B, T, Hk, d = sh.batch, sh.n_tokens, sh.n_kv_heads, sh.head_dim
    k = torch.empty(B, T, Hk, d, dtype=st, device=dev)
    v = torch.empty(B, T, Hk, d, dtype=st, device=dev)
    for b in range(B):
        kb, vb = synth.layer_kv(sh, basis, w, 0, b, device=dev, compute_dtype=torch.float32)
        k[b] = kb
        v[b] = vb
    td = {"basis": basis.to(st).to(dev), "w1": w[0].to(st).to(dev), "b1": w[1].to(st).to(dev),
          "w2": w[2].to(st).to(dev), "b2": w[3].to(st).to(dev)}
    cfg = L.make_config(sh)
    ctx = L.Context(cfg)
    cache = L.alloc_cache(cfg, dev)
    params = L.layer_params(*(td[n] for n in ("basis", "w1", "b1", "w2", "b2")))
    ws = torch.empty(L.workspace_size(cfg, L.OP_ENCODE), dtype=torch.uint8, device=dev)
    L.encode(ctx, k, v, params, cache, ws)
    assert ctx.last_error() == L.OK
    del ws
    return sh, ctx, cfg, cache, td, params, k, v


def sampled_pairs(sh):
    """Eight (batch, KV head) pairs spread over the batch and the heads."""
    B, Hk = sh.batch, sh.n_kv_heads
    return sorted({(i * B // 8, (3 * i + i // 4) % Hk) for i in range(8)} | {(B - 1, Hk - 1)})


def test_encode_properties_and_sampled_errors(full_layer):
    sh, ctx, cfg, cache, td, params, k, v = full_layer
    ridx = cache["res_idx"].cpu().numpy()
    ptr = cache["chunk_ptr"].cpu().numpy()
    assert ridx.shape[-1] == sh.n_res
    assert np.all(np.diff(ridx, axis=-1) > 0) and ridx.min() >= 0 and ridx.max() < sh.n_tokens
    for b in range(sh.batch):
        for h in range(sh.n_kv_heads):
            cnt = np.bincount(ridx[b, h] // sh.chunk, minlength=sh.n_chunks)
            assert np.array_equal(np.diff(ptr[b, h]), cnt) and ptr[b, h, 0] == 0
    rng = np.random.default_rng(0)
    basis = H.f64(td["basis"])
    w1, b1, w2, b2 = (H.f64(td[n]) for n in ("w1", "b1", "w2", "b2"))
    d = sh.head_dim
    for b, h in sampled_pairs(sh):
        toks = np.sort(rng.choice(sh.n_tokens, 96, replace=False))
        kt = H.f64(k[b, toks])                                     # [n, H, d]
        vt = H.f64(v[b, toks, h])
        kp = O.rope_rotate(kt, toks[:, None], sh.theta, inverse=True).reshape(len(toks), -1)
        c = O.project_keys(kp, basis)
        # stored coefficients: the fp64 projection rounds to them, or to a neighbour when
        # the fp32 sum lies within its own error of a rounding midpoint; that error (2048
        # exact products summed in fp32) is ~1e-6 of the row's largest coefficient, which
        # matters only for coefficients near zero
        cg = H.f64(cache["coef"][b, toks])
        cst = O.round_to_storage(c, O.STORE_BF16)
        bound = 2.0 ** (np.floor(np.log2(np.abs(cst) + 1e-30)) - 7) + \
            1e-5 * np.abs(c).max(axis=1, keepdims=True)
        excess = np.abs(cg - cst) - bound
        assert np.all(excess <= 0), (b, h, float(excess.max()),
                                     float(np.abs(c).flat[np.argmax(excess)]))
        e = ((vt - O.predictor(O.rebuild_keys(c, basis, h, d), w1[h], b1[h], w2[h], b2[h],
                               sh.act)) ** 2).sum(-1)
        picked = np.isin(toks, ridx[b, h])
        if picked.any() and (~picked).any():
            lo_in, hi_out = e[picked].min(), e[~picked].max()
            assert lo_in >= hi_out * (1 - 1e-5), (b, h, lo_in, hi_out)


def test_decode_sampled_pairs_match_oracle(L, full_layer):
    sh, ctx, cfg, cache, td, params, k, v = full_layer
    dev = k.device
    kk = min(sh.top_k, sh.n_chunks)
    ws = torch.empty(L.workspace_size(cfg, L.OP_DECODE), dtype=torch.uint8, device=dev)
    G, d = sh.group, sh.head_dim
    basis = H.f64(td["basis"])
    w1, b1, w2, b2 = (H.f64(td[n]) for n in ("w1", "b1", "w2", "b2"))
    pairs = sampled_pairs(sh)
    subs = {}
    for b, h in pairs:
        subs[b, h] = {
            "coef": H.f64(cache["coef"][b:b + 1]),
            "landmark": H.f64(cache["landmark"][b:b + 1, h:h + 1]),
            "res_idx": cache["res_idx"][b:b + 1, h:h + 1].cpu().numpy().astype(np.int64),
            "res_val": H.f64(cache["res_val"][b:b + 1, h:h + 1]),
            "chunk_ptr": cache["chunk_ptr"][b:b + 1, h:h + 1].cpu().numpy().astype(np.int64)}
    ties = 0
    worst = 0.0
    for step in range(2):
        q = synth.queries(sh, 0, step).to(dev)
        out = torch.empty_like(q)
        sel = torch.empty(sh.batch, sh.n_kv_heads, kk, dtype=torch.int32, device=dev)
        L.decode_step(ctx, cache, params, q, out, ws, sel_out=sel)
        assert ctx.last_error() == L.OK
        for b, h in pairs:
            sub = subs[b, h]
            qb = H.f64(q[b:b + 1, h * G:(h + 1) * G])
            osel, scores = O.select_chunks(qb, sub["landmark"], sh.top_k)
            gsel = sel[b:b + 1, h:h + 1].cpu().numpy()
            ties += H.compare_selection(gsel, osel, scores, kk)
            want, _ = O.decode_step(qb, sub, basis[h * d:(h + 1) * d], w1[h:h + 1],
                                    b1[h:h + 1], w2[h:h + 1], b2[h:h + 1], chunk=sh.chunk,
                                    top_k=sh.top_k, theta=sh.theta, act=sh.act,
                                    sel=gsel.astype(np.int64))
            err = H.rel_err(H.f64(out[b:b + 1, h * G:(h + 1) * G]), want)
            worst = max(worst, err)
            assert err <= 2e-2, (step, b, h, err)
        # properties over all pairs: selections ascending, in range, distinct
        s = sel.cpu().numpy()
        assert np.all(np.diff(s, axis=-1) > 0) and s.min() >= 0 and s.max() < sh.n_chunks
        assert torch.isfinite(out.float()).all()
    print(f"{sh.name}: sampled max rel err {worst:.3e}")
    H.assert_ties_bounded(ties, 2 * len(pairs), f"{sh.name} sampled chunk selection")
