"""LowRAM-Q/EQ composition through the C ABI on the GPU, against the oracle:
eviction of the chunks with the smallest all-head landmark norm (lowram_evict), encode
of what is kept at its original RoPE positions with int4 residual rows (fp16 scale per
32 elements), and decode over that cache on both reconstruct-and-attend kernels.

The method composes with quantisation (residuals stored at low precision) and eviction
(agihunt summary, composition paragraph). Readings: see the oracle's quantize_int4_g32,
eviction_keep and encode_evicted.

Bars: kept chunks and residual tokens bit-exact except near-ties (reported and bounded);
kept keys and values copied exactly; int4 scales within one fp16 step and codes equal
except where the residual sits on a rounding midpoint; rebuilt rows and outputs within
the bf16 tolerances of the other tests."""
import numpy as np
import pytest
import torch

import oracle.lowram_oracle as O
from long_context_decode_02_b200 import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu

SHAPE = synth.CONFIGS[4].replace(name="eq-small", n_tokens=4096, batch=2, seed=41)


@pytest.fixture(scope="module")
def L(cuda_device):
    from long_context_decode_02_b200 import lowram
    return lowram


def codes_of(res_val_u8: np.ndarray) -> np.ndarray:
    """Signed int4 codes from packed bytes (element 2i in the low nibble)."""
    lo = (res_val_u8 & 15).astype(np.int16)
    hi = (res_val_u8 >> 4).astype(np.int16)
    q = np.stack([lo, hi], axis=-1).reshape(*res_val_u8.shape[:-1], -1)
    return np.where(q >= 8, q - 16, q)


@pytest.fixture(scope="module")
def eq_cache(L, cuda_device):
    """Full-prefix keys/values, the GPU's eviction and encode of one layer."""
    sh, dev = SHAPE, cuda_device
    t = H.stored_layer(sh, 0)
    td = {k: v.to(dev) for k, v in t.items()}
    cfg = L.make_config(sh)
    ctx = L.Context(cfg, dev.index or 0)
    B, Hk, d = sh.batch, sh.n_kv_heads, sh.head_dim
    kk = torch.empty(B, sh.n_kept_tokens, Hk, d, dtype=torch.bfloat16, device=dev)
    vk = torch.empty_like(kk)
    cache = L.alloc_cache(cfg, dev)
    ws = torch.empty(L.workspace_size(cfg, L.OP_EVICT), dtype=torch.uint8, device=dev)
    L.evict(ctx, td["k"], td["v"], kk, vk, cache["chunk_pos"], ws)
    params = L.layer_params(*(td[n] for n in ("basis", "w1", "b1", "w2", "b2")))
    wse = torch.empty(L.workspace_size(cfg, L.OP_ENCODE), dtype=torch.uint8, device=dev)
    L.encode(ctx, kk, vk, params, cache, wse)
    assert ctx.last_error() == L.OK
    return sh, ctx, cfg, cache, params, t, td, kk, vk


def test_eviction_keeps_largest_landmark_norms(eq_cache):
    sh, ctx, cfg, cache, params, t, td, kk, vk = eq_cache
    pos = cache["chunk_pos"].cpu().numpy()
    # the oracle's eviction on the landmarks as stored in bf16 (its own fp64 means)
    lm = O.round_to_storage(O.chunk_landmarks(H.f64(t["k"]), sh.chunk), O.STORE_BF16)
    want = np.stack([O.eviction_keep(lm[b], sh.n_kept_chunks) for b in range(sh.batch)])
    norms = (lm * lm).sum(axis=(1, 3))                               # [B, N_c full]
    ties = H.compare_selection(pos, want, norms, sh.n_kept_chunks)
    H.assert_ties_bounded(ties, sh.batch, "eviction")
    # the kept rows are copied exactly, at the kept chunks' original rows
    rows = (pos[:, :, None] * sh.chunk + np.arange(sh.chunk)).reshape(sh.batch, -1)
    for b in range(sh.batch):
        assert torch.equal(kk[b].cpu(), t["k"][b, rows[b]])
        assert torch.equal(vk[b].cpu(), t["v"][b, rows[b]])


def test_encode_int4_at_original_positions(eq_cache):
    sh, ctx, cfg, cache, params, t, td, kk, vk = eq_cache
    pos = cache["chunk_pos"].cpu().numpy().astype(np.int64)
    rows = (pos[:, :, None] * sh.chunk + np.arange(sh.chunk)).reshape(sh.batch, -1)
    p = H.oracle_params(t)
    enc = O.encode(H.f64(kk), H.f64(vk), p["basis"], p["w1"], p["b1"], p["w2"], p["b2"],
                   chunk=sh.chunk, n_res=sh.n_res, theta=sh.theta, act=sh.act,
                   store=O.STORE_BF16, positions=rows, res_format="int4")
    # coefficients (RoPE inverted at the original positions) and landmarks
    for name in ("coef", "landmark"):
        g, w = H.f64(cache[name]), enc[name]
        bound = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(w), 1e-30))) - 7) * 1.01 + 1e-6 * np.abs(w).max()
        assert np.all(np.abs(g - w) <= bound), name
    got_idx = cache["res_idx"].cpu().numpy()
    ties = H.compare_selection(got_idx, enc["res_idx"], enc["err"], sh.n_res)
    H.assert_ties_bounded(ties, sh.batch * sh.n_kv_heads, "int4 encode residual pick")
    # int4 rows of the GPU's picked tokens against the exact residual of its stored coef
    gq = codes_of(cache["res_val"].cpu().numpy())
    gs = cache["res_scale"].cpu().numpy().astype(np.float64)
    gcoef = H.f64(cache["coef"])
    v64 = H.f64(vk)
    d = sh.head_dim
    n_scale_diff = n_code_tie = 0
    for b in range(sh.batch):
        for h in range(sh.n_kv_heads):
            idx = got_idx[b, h]
            r = v64[b, idx, h] - O.predictor(O.rebuild_keys(gcoef[b, idx], p["basis"], h, d),
                                             p["w1"][h], p["b1"][h], p["w2"][h], p["b2"][h],
                                             sh.act)
            oq, osc = O.quantize_int4_g32(r)
            # scales: the same fp16 value, or its neighbour when max|R|/7 lies within the
            # GPU residual's error (~1e-5 relative, fp32 accumulation) of an fp16 midpoint
            ulp16 = 2.0 ** (np.floor(np.log2(np.maximum(osc, 1e-30))) - 10)
            diff = gs[b, h] != osc
            assert np.all(np.abs(gs[b, h] - osc) <= ulp16 * 1.0001), (b, h)
            n_scale_diff += int(diff.sum())
            # every stored value is within half a step (of its own scale) of the exact R
            sg = np.repeat(gs[b, h], 32, axis=-1)
            assert np.all(np.abs(gq[b, h] * sg - r) <= sg / 2 * (1 + 2e-3) + 1e-4 * np.abs(r).max())
            # codes: equal where the scales agree, except on rounding midpoints
            same = np.repeat(~diff, 32, axis=-1)
            x = r / np.repeat(np.where(osc > 0, osc, 1.0), 32, axis=-1)
            frac = np.abs(x - np.floor(x) - 0.5)
            bad = same & (gq[b, h] != oq)
            assert np.all(frac[bad] < 2e-3), (b, h, int(bad.sum()))
            n_code_tie += int(bad.sum())
    groups = sh.batch * sh.n_kv_heads * sh.n_res * d // 32
    print(f"int4 rows: {n_scale_diff} scale neighbours over {groups} groups, "
          f"{n_code_tie} code midpoint differences")
    assert n_scale_diff <= groups // 4


def gpu_cache_to_oracle(cache):
    co = H.cache_to_oracle({k: v for k, v in cache.items() if k in
                            ("coef", "landmark", "res_idx", "chunk_ptr")} |
                           {"res_val": cache["coef"][:0]})
    q = codes_of(cache["res_val"].cpu().numpy())
    co["res_val"] = O.dequantize_int4_g32(q, cache["res_scale"].cpu().numpy().astype(np.float64))
    co["chunk_pos"] = cache["chunk_pos"].cpu().numpy().astype(np.int64)
    return co


@pytest.mark.parametrize("variant", ["tc", "simt"])
def test_decode_over_evicted_int4_cache(L, eq_cache, variant):
    sh, ctx, cfg, cache, params, t, td, kk, vk = eq_cache
    dev = kk.device
    v = L.DECODE_TCGEN05 if variant == "tc" else L.DECODE_SIMT
    cfg2 = L.make_config(sh, decode_variant=v)
    ctx2 = L.Context(cfg2, dev.index or 0)
    ws = torch.empty(L.workspace_size(cfg2, L.OP_DECODE), dtype=torch.uint8, device=dev)
    co = gpu_cache_to_oracle(cache)
    p = H.oracle_params(t)
    k = min(sh.top_k, sh.n_chunks)
    ties, errs = 0, []
    for step in range(2):
        q = synth.queries(sh, 0, step)
        out = torch.empty_like(q, device=dev)
        sel = torch.empty(sh.batch, sh.n_kv_heads, k, dtype=torch.int32, device=dev)
        L.decode_step(ctx2, cache, params, q.to(dev), out, ws, sel_out=sel)
        assert ctx2.last_error() == L.OK
        sel_np = sel.cpu().numpy()
        osel, scores = O.select_chunks(H.f64(q), co["landmark"], sh.top_k)
        ties += H.compare_selection(sel_np, osel, scores, k)
        want, _ = O.decode_step(H.f64(q), co, p["basis"], p["w1"], p["b1"], p["w2"], p["b2"],
                                chunk=sh.chunk, top_k=sh.top_k, theta=sh.theta, act=sh.act,
                                sel=sel_np.astype(np.int64))
        errs.append(H.rel_err(H.f64(out), want))
    ctx2.close()
    print(f"EQ decode {variant}: max rel err {max(errs):.2e}")
    assert max(errs) <= H.TOL["bf16"]
    H.assert_ties_bounded(ties, 2 * sh.batch * sh.n_kv_heads, f"EQ decode {variant}")


def test_rebuilt_rows_at_original_positions(L, eq_cache):
    """lowram_debug_reconstruct on the evicted int4 cache: K~_rot re-rotated at the kept
    chunks' original positions and V~ with the dequantized residual rows, element by
    element against the oracle."""
    sh, ctx, cfg, cache, params, t, td, kk, vk = eq_cache
    dev = kk.device
    co = gpu_cache_to_oracle(cache)
    p = H.oracle_params(t)
    q = synth.queries(sh, 0, 3)
    osel, _ = O.select_chunks(H.f64(q), co["landmark"], sh.top_k)
    sel = torch.from_numpy(osel.astype(np.int32)).contiguous().to(dev)
    rows = sh.batch * sh.n_kv_heads * osel.shape[-1] * sh.chunk
    k_rot = torch.empty(rows, sh.head_dim, device=dev)
    h_act = torch.empty(rows, sh.mlp_hidden, device=dev)
    v_rec = torch.empty(rows, sh.head_dim, device=dev)
    out = torch.empty_like(q, device=dev)
    cfg2 = L.make_config(sh, decode_variant=L.DECODE_TCGEN05)
    ctx2 = L.Context(cfg2, dev.index or 0)
    ws = torch.empty(L.workspace_size(cfg2, L.OP_DECODE), dtype=torch.uint8, device=dev)
    L.debug_reconstruct(ctx2, cache, params, q.to(dev), sel, out, k_rot, h_act, v_rec, ws)
    assert ctx2.last_error() == L.OK
    ctx2.close()
    gk = H.f64(k_rot).reshape(sh.batch, sh.n_kv_heads, -1, sh.head_dim)
    gv = H.f64(v_rec).reshape(sh.batch, sh.n_kv_heads, -1, sh.head_dim)
    ek = ev = 0.0
    for b in range(sh.batch):
        for h in range(sh.n_kv_heads):
            _, ok, ov = O.reconstruct_chunks(
                osel[b, h], co["coef"][b], p["basis"], h, sh.head_dim, sh.chunk,
                co["res_idx"][b, h], co["res_val"][b, h], co["chunk_ptr"][b, h],
                p["w1"][h], p["b1"][h], p["w2"][h], p["b2"][h], sh.act, sh.theta,
                co["chunk_pos"][b])
            ek = max(ek, H.rel_err(gk[b, h], ok))
            ev = max(ev, H.rel_err(gv[b, h], ov))
    print(f"EQ rebuilt rows: k {ek:.2e}  v {ev:.2e}")
    assert ek <= 1e-3 and ev <= 2e-2


def test_end_to_end_eq_against_oracle_pipeline(L, eq_cache):
    """GPU evict + encode + decode against the oracle's encode_evicted + decode (outputs
    only: differently rounded landmarks may move a selection legitimately)."""
    sh, ctx, cfg, cache, params, t, td, kk, vk = eq_cache
    dev = kk.device
    p = H.oracle_params(t)
    enc = O.encode_evicted(H.f64(t["k"]), H.f64(t["v"]), p["basis"], p["w1"], p["b1"],
                           p["w2"], p["b2"], chunk=sh.chunk, keep_frac=sh.keep_frac,
                           res_frac=sh.res_frac, theta=sh.theta, act=sh.act,
                           store=O.STORE_BF16, res_format="int4")
    ws = torch.empty(L.workspace_size(cfg, L.OP_DECODE), dtype=torch.uint8, device=dev)
    for step in range(2):
        q = synth.queries(sh, 0, step + 5)
        out = torch.empty_like(q, device=dev)
        L.decode_step(ctx, cache, params, q.to(dev), out, ws)
        assert ctx.last_error() == L.OK
        want, _ = O.decode_step(H.f64(q), enc, p["basis"], p["w1"], p["b1"], p["w2"], p["b2"],
                                chunk=sh.chunk, top_k=sh.top_k, theta=sh.theta, act=sh.act)
        assert H.rel_err(H.f64(out), want) <= H.TOL["bf16"]


def test_append_block_to_evicted_int4_cache(L, eq_cache):
    """Periodic re-compression on the LowRAM-EQ cache: a block of generated tokens after
    the full prefix, compressed with int4 rows at its true positions, appended to the
    evicted prefix (lowram_append). The result keeps chunk positions (the prefix's kept
    chunks, then the block's), its arrays are the two caches concatenated bit for bit
    (int4 codes and fp16 scales included), and decode over it matches the oracle."""
    sh, ctx, cfg, cache, params, t, td, kk, vk = eq_cache
    dev = kk.device
    P, Tb = sh.n_tokens, 512
    nb = int(sh.res_frac * Tb)
    longer = SHAPE.replace(name="eq-block", n_tokens=P + Tb)
    tl = H.stored_layer(longer, 0)
    kb = tl["k"][:, P:].contiguous().to(dev)
    vb = tl["v"][:, P:].contiguous().to(dev)
    cfg_b = L.make_config(sh, n_tokens=Tb, n_positions=P + Tb, n_res=nb)
    ctx_b = L.Context(cfg_b, dev.index or 0)
    blk = L.alloc_cache(cfg_b, dev)
    blk["chunk_pos"].copy_(torch.arange(P // sh.chunk, (P + Tb) // sh.chunk, dtype=torch.int32,
                                        device=dev).expand(sh.batch, -1))
    ws = torch.empty(L.workspace_size(cfg_b, L.OP_ENCODE), dtype=torch.uint8, device=dev)
    L.encode(ctx_b, kb, vb, params, blk, ws)
    torch.cuda.synchronize()
    assert ctx_b.last_error() == L.OK
    T0 = sh.n_kept_tokens
    cfg_d = L.make_config(sh, n_tokens=T0 + Tb, n_positions=P + Tb, n_res=sh.n_res + nb)
    ctx_d = L.Context(cfg_d, dev.index or 0)
    dst = L.alloc_cache(cfg_d, dev)
    L.append(ctx_d, dst, ctx, cache, ctx_b, blk)
    torch.cuda.synchronize()
    assert ctx_d.last_error() == L.OK
    for name, dim in (("coef", 1), ("landmark", 2), ("res_val", 2), ("res_scale", 2),
                      ("chunk_pos", 1)):
        assert torch.equal(dst[name], torch.cat([cache[name], blk[name]], dim=dim)), name
    assert torch.equal(dst["res_idx"], torch.cat([cache["res_idx"], blk["res_idx"] + T0], dim=2))
    n_p = cache["chunk_ptr"].shape[2] - 1
    assert torch.equal(dst["chunk_ptr"], torch.cat([cache["chunk_ptr"][:, :, :n_p],
                                                    blk["chunk_ptr"] + sh.n_res], dim=2))
    assert torch.equal(dst["landmark_norm"], torch.maximum(cache["landmark_norm"],
                                                           blk["landmark_norm"]))
    # decode over the appended cache against the oracle on the same arrays
    wsd = torch.empty(L.workspace_size(cfg_d, L.OP_DECODE), dtype=torch.uint8, device=dev)
    co = gpu_cache_to_oracle(dst)
    p = H.oracle_params(t)
    k = min(sh.top_k, (T0 + Tb) // sh.chunk)
    q = synth.queries(sh, 0, 5)
    out = torch.empty_like(q, device=dev)
    sel = torch.empty(sh.batch, sh.n_kv_heads, k, dtype=torch.int32, device=dev)
    L.decode_step(ctx_d, dst, params, q.to(dev), out, wsd, sel_out=sel)
    torch.cuda.synchronize()
    assert ctx_d.last_error() == L.OK
    sel_np = sel.cpu().numpy()
    osel, scores = O.select_chunks(H.f64(q), co["landmark"], sh.top_k)
    ties = H.compare_selection(sel_np, osel, scores, k)
    H.assert_ties_bounded(ties, sh.batch * sh.n_kv_heads, "EQ appended-cache decode")
    want, _ = O.decode_step(H.f64(q), co, p["basis"], p["w1"], p["b1"], p["w2"], p["b2"],
                            chunk=sh.chunk, top_k=sh.top_k, theta=sh.theta, act=sh.act,
                            sel=sel_np.astype(np.int64))
    assert H.rel_err(H.f64(out), want) <= H.TOL["bf16"]
