"""Pins of the CPU oracle to things other than itself (closed forms, brute force,
invariants the method's definitions fix, and library routines), plus mutation tests
that plant plausible mistakes in the oracle and check that some pin catches each.

CPU only; sized to run in seconds.
"""
import cmath
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.lowram_oracle as O
from long_context_decode_02_b200 import synth


def _np(t):
    return t.detach().to(torch.float64).cpu().numpy()


def tiny_shape(**kw):
    base = dict(name="pin", batch=2, n_tokens=64, n_layers=1, n_kv_heads=2, n_q_heads=4,
                head_dim=8, rank=16, chunk=4, top_k=16, res_frac=1.0, mlp_hidden=12,
                act=O.ACT_SILU, dtype="f32", theta=1e4, outlier_frac=0.05, steps=1,
                seed=11)
    base.update(kw)
    return synth.Shape(**base)


def make_layer(shape, layer=0):
    """Inputs of one layer in fp64 (keys, values, basis, weights, queries)."""
    basis = synth.group_basis(shape, 0)
    w = synth.layer_weights(shape, layer)
    ks, vs = [], []
    for b in range(shape.batch):
        k, v = synth.layer_kv(shape, basis, w, layer, b)
        ks.append(k)
        vs.append(v)
    k = torch.stack(ks)
    v = torch.stack(vs)
    q = synth.queries(shape, layer, 0)
    return dict(k=_np(k), v=_np(v), basis=_np(basis), w=[_np(t) for t in w], q=_np(q))


# ----------------------------------------------------------------------------------
# pin checks, written against a module object so mutation tests can reuse them
# ----------------------------------------------------------------------------------
def check_rope_closed_form(M):
    d, theta = 16, 1e4
    for i in range(d // 2):
        x = np.zeros(d)
        x[i] = 1.0
        y = M.rope_rotate(x, 1, theta)
        a = theta ** (-2.0 * i / d)
        expect = np.zeros(d)
        expect[i] = math.cos(a)
        expect[i + d // 2] = math.sin(a)
        assert np.allclose(y, expect, atol=1e-15), (i, y, expect)
    # complex-number form at a large position: (x_i + j x_{i+d/2}) e^{j t theta_i}
    rng = np.random.default_rng(0)
    x = rng.standard_normal(d)
    t = 262143
    y = M.rope_rotate(x, t, theta)
    for i in range(d // 2):
        z = complex(x[i], x[i + d // 2]) * cmath.exp(1j * t * theta ** (-2.0 * i / d))
        assert abs(y[i] - z.real) < 1e-9 and abs(y[i + d // 2] - z.imag) < 1e-9


def check_rope_group_properties(M):
    rng = np.random.default_rng(1)
    d, theta = 32, 5e5
    x = rng.standard_normal((5, d))
    pos = np.array([0, 1, 17, 4096, 262143])
    assert np.allclose(M.rope_rotate(x[:1], 0, theta), x[:1], atol=0)      # R(0) = I
    y = M.rope_rotate(x, pos, theta)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)
    assert np.allclose(M.rope_rotate(y, pos, theta, inverse=True), x, atol=1e-13)
    # relative position: <R(m)a, R(n)b> depends on m - n only
    a, b = rng.standard_normal(d), rng.standard_normal(d)
    s1 = M.rope_rotate(a, 100, theta) @ M.rope_rotate(b, 37, theta)
    s2 = M.rope_rotate(a, 1100, theta) @ M.rope_rotate(b, 1037, theta)
    assert abs(s1 - s2) < 1e-10


def check_projection(M):
    rng = np.random.default_rng(2)
    H, d = 3, 8
    D = H * d
    # full rank, square orthogonal basis: rebuild(project(x)) == x for every head
    q_full, _ = np.linalg.qr(rng.standard_normal((D, D)))
    x = rng.standard_normal((10, D))
    c = M.project_keys(x, q_full)
    for h in range(H):
        assert np.allclose(M.rebuild_keys(c, q_full, h, d), x[:, h * d:(h + 1) * d],
                           atol=1e-12)
    # reduced rank: coefficients are the least-squares solution (library routine)
    b_red, _ = np.linalg.qr(rng.standard_normal((D, 7)))
    c = M.project_keys(x, b_red)
    lst, *_ = np.linalg.lstsq(b_red, x.T, rcond=None)
    assert np.allclose(c, lst.T, atol=1e-12)
    full = np.concatenate([M.rebuild_keys(c, b_red, h, d) for h in range(H)], axis=1)
    assert np.allclose(full, lst.T @ b_red.T, atol=1e-12)


def check_landmarks_and_scores(M):
    rng = np.random.default_rng(3)
    B, T, H, d, C, G = 2, 24, 2, 4, 4, 3
    k = rng.standard_normal((B, T, H, d))
    lm = M.chunk_landmarks(k, C)
    assert lm.shape == (B, H, T // C, d)
    for b in range(B):
        for h in range(H):
            for c in range(T // C):
                brute = [math.fsum(k[b, c * C + i, h, j] for i in range(C)) / C
                         for j in range(d)]
                assert np.allclose(lm[b, h, c], brute, atol=1e-15)
    # linearity: q . L_c = mean over the chunk of q . K_t
    q = rng.standard_normal(d)
    assert np.allclose(lm[0, 1] @ q, (k[0, :, 1] @ q).reshape(-1, C).mean(1), atol=1e-14)
    # chunk score = max over the group's heads; a group where one head dominates
    qg = np.zeros((G, d))
    qg[2] = q
    s = M.chunk_scores(qg, lm[1, 0])
    assert np.allclose(s, np.maximum(lm[1, 0] @ q, 0.0), atol=1e-15)
    qg = rng.standard_normal((G, d))
    s = M.chunk_scores(qg, lm[0, 0])
    brute = [max(math.fsum(qg[g, j] * lm[0, 0, c, j] for j in range(d)) for g in range(G))
             for c in range(T // C)]
    assert np.allclose(s, brute, atol=1e-14)


def check_encode_landmarks(M):
    """encode's landmarks are the chunk means of the POST-RoPE keys it is given, per KV
    head (brute-force fsum over the chunk's rows of k_cache), stored unrounded at f64."""
    sh = tiny_shape(res_frac=0.25, rank=6)
    L = make_layer(sh)
    cache = M.encode(L["k"], L["v"], L["basis"], *L["w"], n_res=sh.n_res,
                     store=M.STORE_F64, chunk=sh.chunk, theta=sh.theta, act=sh.act)
    k, C = L["k"], sh.chunk
    assert cache["landmark"].shape == (sh.batch, sh.n_kv_heads, sh.n_chunks, sh.head_dim)
    for b in range(sh.batch):
        for h in range(sh.n_kv_heads):
            for c in range(sh.n_chunks):
                brute = [math.fsum(k[b, c * C + i, h, j] for i in range(C)) / C
                         for j in range(sh.head_dim)]
                assert np.allclose(cache["landmark"][b, h, c], brute, rtol=0, atol=1e-15)


def check_topk(M):
    rng = np.random.default_rng(4)
    for n, k in [(50, 7), (50, 50), (50, 80), (200, 1)]:
        for s in (rng.standard_normal(n), rng.integers(0, 4, n).astype(float)):
            got = M.topk_ascending(s, k)
            brute = sorted(sorted(range(n), key=lambda i: (-s[i], i))[:min(k, n)])
            assert list(got) == brute, (n, k)


def check_predictor(M):
    rng = np.random.default_rng(5)
    d, Fh = 8, 12
    x = rng.standard_normal((9, d))
    w1, b1 = rng.standard_normal((Fh, d)), rng.standard_normal(Fh)
    w2, b2 = rng.standard_normal((d, Fh)), rng.standard_normal(d)
    tx = torch.tensor(x)
    for act, fn in ((M.ACT_SILU, F.silu), (M.ACT_GELU_ERF,
                                           lambda t: F.gelu(t, approximate="none"))):
        ref = F.linear(fn(F.linear(tx, torch.tensor(w1), torch.tensor(b1))),
                       torch.tensor(w2), torch.tensor(b2)).numpy()
        assert np.allclose(M.predictor(x, w1, b1, w2, b2, act), ref, atol=1e-13)


def check_full_rank_exactness(M):
    """Full rank, every token a residual, every chunk selected: decode == dense attention
    over the original keys/values, and encode reconstructs K and V exactly."""
    sh = tiny_shape(rank=16, n_kv_heads=2, head_dim=8, res_frac=1.0, top_k=10 ** 6)
    L = make_layer(sh)
    kw = dict(chunk=sh.chunk, theta=sh.theta, act=sh.act)
    cache = M.encode(L["k"], L["v"], L["basis"], *L["w"], n_res=sh.n_res,
                     store=M.STORE_F64, **kw)
    w1, b1, w2, b2 = L["w"]
    for b in range(sh.batch):
        for h in range(sh.n_kv_heads):
            sel = np.arange(sh.n_chunks)
            toks, k_rot, v_rec = M.reconstruct_chunks(
                sel, cache["coef"][b], L["basis"], h, sh.head_dim, sh.chunk,
                cache["res_idx"][b, h], cache["res_val"][b, h], cache["chunk_ptr"][b, h],
                w1[h], b1[h], w2[h], b2[h], sh.act, sh.theta)
            assert np.allclose(k_rot, L["k"][b, toks, h], atol=1e-12)
            assert np.allclose(v_rec, L["v"][b, toks, h], atol=1e-12)
    out, sel = M.decode_step(L["q"], cache, L["basis"], *L["w"], top_k=sh.top_k, **kw)
    dense = M.dense_attention(L["q"], L["k"], L["v"])
    assert np.allclose(out, dense, atol=1e-12)
    # and the dense textbook form equals torch's attention routine
    G = sh.group
    tq = torch.tensor(L["q"])[:, :, None, :]                          # [B, Hq, 1, d]
    tk = torch.tensor(L["k"]).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    tv = torch.tensor(L["v"]).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    ref = F.scaled_dot_product_attention(tq, tk, tv)[:, :, 0, :].numpy()
    assert np.allclose(dense, ref, atol=1e-12)


def check_residual_pick(M):
    sh = synth.CONFIGS[0].replace(n_layers=1, n_tokens=512)
    L = make_layer(sh)
    kw = dict(chunk=sh.chunk, theta=sh.theta, act=sh.act)
    c64 = M.encode(L["k"], L["v"], L["basis"], *L["w"], n_res=sh.n_res,
                   store=M.STORE_F64, **kw)
    cbf = M.encode(L["k"], L["v"], L["basis"], *L["w"], n_res=sh.n_res,
                   store=M.STORE_BF16, **kw)
    # errors use the unrounded coefficients: independent of the storage precision
    assert np.array_equal(c64["err"], cbf["err"])
    d = sh.head_dim
    w1, b1, w2, b2 = L["w"]
    for h in range(sh.n_kv_heads):
        e = c64["err"][0, h]
        # brute force: per-token squared error, then a full sort
        brute_e = []
        for t in range(sh.n_tokens):
            kp = M.rope_rotate(L["k"][0, t], t, sh.theta, inverse=True).reshape(-1)
            ct = L["basis"].T @ kp
            vhat = M.predictor(L["basis"][h * d:(h + 1) * d] @ ct, w1[h], b1[h], w2[h],
                               b2[h], sh.act)
            brute_e.append(math.fsum((L["v"][0, t, h] - vhat) ** 2))
        assert np.allclose(e, brute_e, rtol=1e-12)
        order = sorted(range(sh.n_tokens), key=lambda t: (-brute_e[t], t))[:sh.n_res]
        assert list(c64["res_idx"][0, h]) == sorted(order)
        # every planted outlier row is among the residuals (error ~ d*9 >> noise)
        n_out = int(sh.outlier_frac * sh.n_tokens)
        big = np.argsort(-np.abs(L["v"][0, :, h]).max(axis=1))[:n_out]
        assert set(big.tolist()) <= set(c64["res_idx"][0, h].tolist())
        # CSR offsets count the residual rows of every chunk
        ptr = c64["chunk_ptr"][0, h]
        for c in range(sh.n_chunks):
            n_in = sum(1 for t in c64["res_idx"][0, h] if c * sh.chunk <= t < (c + 1) * sh.chunk)
            assert ptr[c + 1] - ptr[c] == n_in
        # the stored residual restores V up to its own rounding: it was taken against
        # the predictor run on the STORED coefficients
        idx = cbf["res_idx"][0, h]
        vhat_s = M.predictor(M.rebuild_keys(cbf["coef"][0, idx], L["basis"], h, d),
                             w1[h], b1[h], w2[h], b2[h], sh.act)
        exact_r = L["v"][0, idx, h] - vhat_s
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact_r), 1e-300))) - 7)
        assert np.all(np.abs(vhat_s + cbf["res_val"][0, h] - L["v"][0, idx, h])
                      <= 0.5 * ulp + 1e-15)


def check_selection_and_edges(M):
    sh = tiny_shape(res_frac=0.25, top_k=5, rank=6)
    L = make_layer(sh)
    kw = dict(chunk=sh.chunk, theta=sh.theta, act=sh.act)
    cache = M.encode(L["k"], L["v"], L["basis"], *L["w"], n_res=sh.n_res,
                     store=M.STORE_F32, **kw)
    out, sel = M.decode_step(L["q"], cache, L["basis"], *L["w"], top_k=sh.top_k, **kw)
    G = sh.group
    for b in range(sh.batch):
        for h in range(sh.n_kv_heads):
            s = [max(float(L["q"][b, h * G + g] @ cache["landmark"][b, h, c])
                     for g in range(G)) for c in range(sh.n_chunks)]
            brute = sorted(sorted(range(sh.n_chunks), key=lambda c: (-s[c], c))[:sh.top_k])
            assert list(sel[b, h]) == brute
    # the output is a convex combination of reconstructed values: bounded by them
    # no residuals at all: a valid cache, decode still runs
    c0 = M.encode(L["k"], L["v"], L["basis"], *L["w"], n_res=0, store=M.STORE_F32, **kw)
    assert c0["res_idx"].shape[-1] == 0 and np.all(c0["chunk_ptr"] == 0)
    out0, _ = M.decode_step(L["q"], c0, L["basis"], *L["w"], top_k=1, **kw)
    assert np.all(np.isfinite(out0))


def check_cholesky_qr(M):
    """Cholesky-QR is the thin QR factorisation with a positive diagonal in R: equal to
    numpy's QR (a library routine) once the signs of its R diagonal are fixed."""
    rng = np.random.default_rng(21)
    y = rng.standard_normal((40, 7)) @ np.diag([5, 4, 3, 2, 1, 0.5, 0.25])
    q = M.cholesky_qr(y)
    qn, rn = np.linalg.qr(y)
    qn = qn * np.sign(np.diag(rn))
    assert np.allclose(q, qn, atol=1e-10)
    assert np.allclose(q.T @ q, np.eye(7), atol=1e-12)


def check_fit_basis(M):
    """The randomised range finder returns the top-r right singular subspace of the key
    rows: exactly for an exactly rank-r matrix, exactly (via Rayleigh-Ritz) when the test
    matrix spans everything, and to numpy's SVD (a library routine) with oversampling."""
    rng = np.random.default_rng(22)
    D, r, N = 32, 5, 400
    sig = np.array([10.0, 8.0, 6.0, 5.0, 4.0])
    # planted exact rank r, no oversampling (Cholesky-QR needs full column rank)
    V, _ = np.linalg.qr(rng.standard_normal((D, r)))
    A = (rng.standard_normal((N, r)) * sig) @ V.T
    B = M.fit_basis(A, r, rng.standard_normal((D, r)))
    assert B.shape == (D, r)
    assert np.allclose(B.T @ B, np.eye(r), atol=1e-12)
    assert np.allclose(B @ B.T, V @ V.T, atol=1e-12)
    # a full-width test matrix and no power step: Rayleigh-Ritz over all of R^D gives the
    # SVD subspace exactly even though the spectrum has no real gap
    Vf, _ = np.linalg.qr(rng.standard_normal((D, D)))
    A = (rng.standard_normal((N, D)) * np.linspace(4.0, 1.0, D)) @ Vf.T
    vr = np.linalg.svd(A, full_matrices=False)[2][:r].T
    B = M.fit_basis(A, r, rng.standard_normal((D, D)), n_power=0)
    assert np.allclose(B @ B.T, vr @ vr.T, atol=1e-10)
    # oversampled, noisy, with a gap
    A = (rng.standard_normal((N, r)) * sig) @ V.T + 0.01 * rng.standard_normal((N, D))
    vr = np.linalg.svd(A, full_matrices=False)[2][:r].T
    B = M.fit_basis(A, r, rng.standard_normal((D, r + 4)))
    assert np.allclose(B @ B.T, vr @ vr.T, atol=1e-8)


def check_fit_basis_recovers_generator(M):
    """Fitted on the pre-RoPE keys of a synthetic two-layer group (keys = c B_g^T +
    0.05 noise), the basis spans the generator's B_g to within the noise."""
    sh = tiny_shape(n_tokens=256, n_layers=2, rank=5, res_frac=0.1)
    basis = synth.group_basis(sh, 0)
    rows = []
    for layer in range(2):
        w = synth.layer_weights(sh, layer)
        for b in range(sh.batch):
            k, _ = synth.layer_kv(sh, basis, w, layer, b)
            k = _np(k)
            pos = np.arange(k.shape[0])[:, None]
            rows.append(M.rope_rotate(k, pos, sh.theta, inverse=True).reshape(k.shape[0], -1))
    a = np.concatenate(rows)
    rng = np.random.default_rng(23)
    B = M.fit_basis(a, sh.rank, rng.standard_normal((a.shape[1], sh.rank + 4)))
    bg = _np(basis)
    assert np.linalg.norm(B @ B.T - bg @ bg.T, 2) < 0.03


def check_int4_quantize(M):
    """int4 codes with an fp16 scale per 32 elements: exact on grids of fp16 multiples,
    half a step at most elsewhere, ties to even, zero groups, and the fp16 rounding
    itself against torch's conversion (a library routine)."""
    rng = np.random.default_rng(31)
    # rows whose groups are exact multiples of an fp16 step, with a +-7 step present
    steps = np.float16(rng.uniform(0.01, 2.0, (5, 4))).astype(np.float64)
    ints = rng.integers(-7, 8, (5, 4, 32))
    ints[:, :, 0] = np.where(rng.random((5, 4)) < 0.5, 7, -7)
    x = (ints * steps[..., None]).reshape(5, 128)
    q, s = M.quantize_int4_g32(x)
    assert np.array_equal(s, steps)
    assert np.array_equal(q.reshape(5, 4, 32), ints)
    assert np.array_equal(M.dequantize_int4_g32(q, s), x)
    # arbitrary rows: within half a step, codes in range, the largest element at +-7
    x = rng.standard_normal((50, 128)) * 10.0 ** rng.integers(-3, 3, (50, 1))
    q, s = M.quantize_int4_g32(x)
    err = np.abs(M.dequantize_int4_g32(q, s) - x).reshape(50, 4, 32)
    assert np.all(err <= s[..., None] / 2 * (1 + 1e-12))
    assert q.min() >= -8 and q.max() <= 7
    g = np.abs(x).reshape(50, 4, 32)
    top = np.take_along_axis(np.abs(q).reshape(50, 4, 32), g.argmax(-1)[..., None], -1)
    assert np.all(top == 7)
    # ties to even: x / s = 2.5 -> 2, 3.5 -> 4, -2.5 -> -2, -0.5 -> 0
    row = np.zeros(32)
    row[:5] = [7.0, 2.5, 3.5, -2.5, -0.5]
    q, s = M.quantize_int4_g32(row)
    assert s[0] == 1.0 and list(q[:5]) == [7, 2, 4, -2, 0]
    # an all-zero group has scale 0 and codes 0
    q, s = M.quantize_int4_g32(np.zeros(64))
    assert np.all(s == 0) and np.all(q == 0)
    # fp16 rounding of fp32 values (torch converts those with one rounding; from fp64 it
    # rounds through fp32 first, which is not a reference for fp64 inputs)
    y = (rng.standard_normal(4000) * 10.0 ** rng.integers(-6, 4, 4000)).astype(np.float32)
    y[:3] = [1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2048.0 + 1.0]   # ties
    ref = torch.from_numpy(y).to(torch.float16).to(torch.float64).numpy()
    assert np.array_equal(M.f64_to_f16(y.astype(np.float64)), ref)
    assert M.f64_to_f16(np.array([1.0 + 2.0 ** -11 + 2.0 ** -40]))[0] == 1.0 + 2.0 ** -10


def check_eviction(M):
    """The kept chunks are those with the largest all-head landmark norm, ties to the
    lower chunk index (brute force: fsum of squares, Python sort), ascending."""
    rng = np.random.default_rng(32)
    H, n, d = 3, 40, 8
    lm = rng.standard_normal((H, n, d))
    lm[:, 7] = lm[:, 3]            # exact ties in norm
    lm[:, 30] = -lm[:, 3]
    for n_keep in (1, 13, 20, 40):
        norm = [math.fsum(float(lm[h, c, j]) ** 2 for h in range(H) for j in range(d))
                for c in range(n)]
        brute = sorted(sorted(range(n), key=lambda c: (-norm[c], c))[:n_keep])
        assert list(M.eviction_keep(lm, n_keep)) == brute, n_keep


def check_evicted_full_rank_exactness(M):
    """Eviction of half the chunks, then full rank, every kept token a residual and every
    kept chunk selected (f64 storage): decode equals dense attention over the kept
    tokens' original keys and values, at their original positions."""
    sh = tiny_shape(rank=16, n_kv_heads=2, head_dim=8, res_frac=1.0, top_k=10 ** 6,
                    n_tokens=64, chunk=4)
    L = make_layer(sh)
    kw = dict(chunk=sh.chunk, theta=sh.theta, act=sh.act)
    cache = M.encode_evicted(L["k"], L["v"], L["basis"], *L["w"], keep_frac=0.5,
                             res_frac=1.0, store=M.STORE_F64, **kw)
    pos = cache["chunk_pos"]
    assert pos.shape == (sh.batch, sh.n_chunks // 2)
    rows = (pos[:, :, None] * sh.chunk + np.arange(sh.chunk)).reshape(sh.batch, -1)
    kk = np.stack([L["k"][b, rows[b]] for b in range(sh.batch)])
    vv = np.stack([L["v"][b, rows[b]] for b in range(sh.batch)])
    out, _ = M.decode_step(L["q"], cache, L["basis"], *L["w"], top_k=sh.top_k, **kw)
    assert np.allclose(out, M.dense_attention(L["q"], kk, vv), atol=1e-12)
    # the eviction kept the largest all-head landmark norms of the stored landmarks
    for b in range(sh.batch):
        nrm = (cache["full_landmark"][b] ** 2).sum(axis=(0, 2))
        assert nrm[pos[b]].min() >= np.delete(nrm, pos[b]).max()


def check_int4_residual_encode(M):
    """encode with int4 residual rows: res_val is the dequantized code, and the stored
    prediction plus it restores V within half a quantisation step per element."""
    sh = synth.CONFIGS[0].replace(n_layers=1, n_tokens=256)
    L = make_layer(sh)
    cache = M.encode(L["k"], L["v"], L["basis"], *L["w"], chunk=sh.chunk, n_res=sh.n_res,
                     theta=sh.theta, act=sh.act, store=M.STORE_BF16, res_format="int4")
    assert np.array_equal(cache["res_val"],
                          M.dequantize_int4_g32(cache["res_q"], cache["res_scale"]))
    w1, b1, w2, b2 = L["w"]
    d = sh.head_dim
    for h in range(sh.n_kv_heads):
        idx = cache["res_idx"][0, h]
        vhat = M.predictor(M.rebuild_keys(cache["coef"][0, idx], L["basis"], h, d),
                           w1[h], b1[h], w2[h], b2[h], sh.act)
        err = np.abs(vhat + cache["res_val"][0, h] - L["v"][0, idx, h]).reshape(len(idx), -1, 32)
        assert np.all(err <= cache["res_scale"][0, h][..., None] / 2 * (1 + 1e-9) + 1e-12)


def check_suffix_decode(M):
    """Compressed prefix + uncompressed suffix, one softmax: at full rank, every token a
    residual and every chunk selected, it equals dense attention over the prefix's and
    the suffix's keys and values together; an empty suffix leaves decode unchanged."""
    sh = tiny_shape(rank=16, n_kv_heads=2, head_dim=8, res_frac=1.0, top_k=10 ** 6)
    L = make_layer(sh)
    kw = dict(chunk=sh.chunk, theta=sh.theta, act=sh.act)
    cache = M.encode(L["k"], L["v"], L["basis"], *L["w"], n_res=sh.n_res,
                     store=M.STORE_F64, **kw)
    rng = np.random.default_rng(33)
    S = 11
    ks = rng.standard_normal((sh.batch, S, sh.n_kv_heads, sh.head_dim))
    vs = rng.standard_normal((sh.batch, S, sh.n_kv_heads, sh.head_dim))
    out, _ = M.decode_step_with_suffix(L["q"], cache, L["basis"], *L["w"], ks, vs,
                                       top_k=sh.top_k, **kw)
    dense = M.dense_attention(L["q"], np.concatenate([L["k"], ks], axis=1),
                              np.concatenate([L["v"], vs], axis=1))
    assert np.allclose(out, dense, atol=1e-12)
    sh2 = tiny_shape(res_frac=0.25, top_k=5, rank=6)
    L2 = make_layer(sh2)
    c2 = M.encode(L2["k"], L2["v"], L2["basis"], *L2["w"], n_res=sh2.n_res,
                  store=M.STORE_F32, chunk=sh2.chunk, theta=sh2.theta, act=sh2.act)
    empty = np.zeros((sh2.batch, 0, sh2.n_kv_heads, sh2.head_dim))
    a, _ = M.decode_step_with_suffix(L2["q"], c2, L2["basis"], *L2["w"], empty, empty,
                                     chunk=sh2.chunk, top_k=sh2.top_k, theta=sh2.theta,
                                     act=sh2.act)
    b_, _ = M.decode_step(L2["q"], c2, L2["basis"], *L2["w"], chunk=sh2.chunk,
                          top_k=sh2.top_k, theta=sh2.theta, act=sh2.act)
    assert np.allclose(a, b_, atol=1e-14)


def _block_errors_brute(k_block, v_block, basis, w, first, theta, act, h):
    """Squared predictor errors of a block's tokens for head h, written out per token
    with RoPE undone through complex numbers (pairs (i, i + d/2) as x + iy)."""
    w1, b1, w2, b2 = w
    B, Tb, H, d = k_block.shape
    half = d // 2
    inv = theta ** (-2.0 * np.arange(half) / d)
    out = np.empty((B, Tb))
    for b in range(B):
        for t in range(Tb):
            rows = []
            for hh in range(H):
                z = (k_block[b, t, hh, :half] + 1j * k_block[b, t, hh, half:]) * np.exp(
                    -1j * (first + t) * inv)
                rows.append(np.concatenate([z.real, z.imag]))
            c = basis.T @ np.concatenate(rows)
            x = basis[h * d:(h + 1) * d] @ c
            pre = w1[h] @ x + b1[h]
            a = pre / (1.0 + np.exp(-pre)) if act == O.ACT_SILU else 0.5 * pre * (
                1.0 + np.vectorize(math.erf)(pre / math.sqrt(2.0)))
            vh = w2[h] @ a + b2[h]
            out[b, t] = float(((v_block[b, t, h] - vh) ** 2).sum())
    return out


def check_block_append(M):
    """Periodic re-compression: a block of whole chunks compressed at its true positions
    and appended after the compressed prefix. (1) Full rank, every token a residual and
    every chunk selected: decode equals dense attention over prefix and block together,
    also after eviction of half the prefix's chunks. (2) The block's residual rows are
    its own largest-error tokens (errors written out per token), moved past the prefix's
    rows; the CSR counts each chunk's rows."""
    sh = tiny_shape(rank=16, n_kv_heads=2, head_dim=8, res_frac=1.0, top_k=10 ** 6)
    L = make_layer(sh)
    kw = dict(chunk=sh.chunk, theta=sh.theta, act=sh.act)
    T0 = 48
    pre = M.encode(L["k"][:, :T0], L["v"][:, :T0], L["basis"], *L["w"], n_res=T0,
                   store=M.STORE_F64, **kw)
    blk = M.encode_block(L["k"][:, T0:], L["v"][:, T0:], L["basis"], *L["w"],
                         n_res=sh.n_tokens - T0, store=M.STORE_F64, first_position=T0, **kw)
    cat = M.append_block(pre, blk, prefix_tokens=T0, chunk=sh.chunk,
                         block_first_chunk=T0 // sh.chunk)
    assert cat.get("chunk_pos") is None
    out, _ = M.decode_step(L["q"], cat, L["basis"], *L["w"], top_k=sh.top_k, **kw)
    assert np.allclose(out, M.dense_attention(L["q"], L["k"], L["v"]), atol=1e-12)
    # an evicted prefix (half its chunks kept) followed by the block
    ev = M.encode_evicted(L["k"][:, :T0], L["v"][:, :T0], L["basis"], *L["w"], keep_frac=0.5,
                          res_frac=1.0, store=M.STORE_F64, **kw)
    cat2 = M.append_block(ev, blk, prefix_tokens=T0 // 2, chunk=sh.chunk,
                          block_first_chunk=T0 // sh.chunk)
    rows = (ev["chunk_pos"][:, :, None] * sh.chunk + np.arange(sh.chunk)).reshape(sh.batch, -1)
    kk = np.stack([np.concatenate([L["k"][b, rows[b]], L["k"][b, T0:]]) for b in range(sh.batch)])
    vv = np.stack([np.concatenate([L["v"][b, rows[b]], L["v"][b, T0:]]) for b in range(sh.batch)])
    out2, _ = M.decode_step(L["q"], cat2, L["basis"], *L["w"], top_k=sh.top_k, **kw)
    assert np.allclose(out2, M.dense_attention(L["q"], kk, vv), atol=1e-12)
    # (2) a quarter of each part's tokens residual
    sh2 = tiny_shape(res_frac=0.25, rank=6, top_k=5)
    L2 = make_layer(sh2)
    kw2 = dict(chunk=sh2.chunk, theta=sh2.theta, act=sh2.act)
    nb = (sh2.n_tokens - T0) // 4
    pre2 = M.encode(L2["k"][:, :T0], L2["v"][:, :T0], L2["basis"], *L2["w"], n_res=T0 // 4,
                    store=M.STORE_F32, **kw2)
    blk2 = M.encode_block(L2["k"][:, T0:], L2["v"][:, T0:], L2["basis"], *L2["w"], n_res=nb,
                          store=M.STORE_F32, first_position=T0, **kw2)
    cat3 = M.append_block(pre2, blk2, prefix_tokens=T0, chunk=sh2.chunk,
                          block_first_chunk=T0 // sh2.chunk)
    for h in range(sh2.n_kv_heads):
        e = _block_errors_brute(L2["k"][:, T0:], L2["v"][:, T0:], L2["basis"], L2["w"], T0,
                                sh2.theta, sh2.act, h)
        for b in range(sh2.batch):
            want = np.sort(np.argsort(-e[b], kind="stable")[:nb]) + T0
            assert np.array_equal(cat3["res_idx"][b, h, T0 // 4:], want)
            assert np.array_equal(cat3["res_idx"][b, h, :T0 // 4], pre2["res_idx"][b, h])
            counts = np.bincount(cat3["res_idx"][b, h] // sh2.chunk,
                                 minlength=sh2.n_tokens // sh2.chunk)
            assert np.array_equal(np.diff(cat3["chunk_ptr"][b, h]), counts)
            assert cat3["chunk_ptr"][b, h, 0] == 0
    assert np.array_equal(cat3["res_val"][:, :, T0 // 4:], blk2["res_val"])


ALL_CHECKS = [check_rope_closed_form, check_rope_group_properties, check_projection,
              check_landmarks_and_scores, check_encode_landmarks, check_topk, check_predictor,
              check_full_rank_exactness, check_residual_pick, check_selection_and_edges,
              check_cholesky_qr, check_fit_basis, check_fit_basis_recovers_generator,
              check_int4_quantize, check_eviction, check_evicted_full_rank_exactness,
              check_int4_residual_encode, check_suffix_decode, check_block_append]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(O)


def test_bf16_rounding_matches_torch_and_ties_to_even():
    rng = np.random.default_rng(7)
    x32 = (rng.standard_normal(10000) * 10.0 ** rng.integers(-6, 6, 10000)).astype(np.float32)
    ours = O.f64_to_bf16_bits(x32.astype(np.float64))
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    one = 1.0
    assert O.f64_to_bf16_bits(np.array([one]))[0] == 0x3F80
    assert O.f64_to_bf16_bits(np.array([one + 2.0 ** -8]))[0] == 0x3F80       # tie -> even
    assert O.f64_to_bf16_bits(np.array([one + 3 * 2.0 ** -8]))[0] == 0x3F82   # tie -> even
    assert O.f64_to_bf16_bits(np.array([one + 2.0 ** -8 + 2.0 ** -30]))[0] == 0x3F81


def test_reorder_identity_fp64():
    """The library applies W2 after the attention sum; in exact arithmetic this equals
    attending over the predicted values (softmax weights sum to one)."""
    rng = np.random.default_rng(8)
    n, d, Fh = 40, 8, 12
    kp = rng.standard_normal((n, d))
    w1, b1 = rng.standard_normal((Fh, d)), rng.standard_normal(Fh)
    w2, b2 = rng.standard_normal((d, Fh)), rng.standard_normal(d)
    r = np.zeros((n, d))
    r[::3] = rng.standard_normal((len(range(0, n, 3)), d))
    z = rng.standard_normal(n)
    p = np.exp(z - z.max())
    plain = (p / p.sum()) @ (O.predictor(kp, w1, b1, w2, b2, O.ACT_SILU) + r)
    hid = O.activation(kp @ w1.T + b1, O.ACT_SILU)
    reorder = (w2 @ (p @ hid) + p @ r) / p.sum() + b2
    assert np.allclose(plain, reorder, atol=1e-12)


# ----------------------------------------------------------------------------------
# mutation tests: plant a plausible mistake in the oracle; some pin must fail
# ----------------------------------------------------------------------------------
def _fails(check, monkeypatch, name, bad):
    monkeypatch.setattr(O, name, bad)
    with pytest.raises(AssertionError):
        check(O)


def test_mutation_rope_wrong_sign(monkeypatch):
    orig = O.rope_rotate
    _fails(lambda M: (check_rope_closed_form(M)), monkeypatch, "rope_rotate",
           lambda x, pos, theta, inverse=False: orig(x, pos, theta, not inverse))


def test_mutation_rope_not_reapplied(monkeypatch):
    orig = O.rope_rotate

    def bad(x, pos, theta, inverse=False):
        return orig(x, pos, theta, True) if inverse else np.asarray(x, np.float64)
    _fails(check_full_rank_exactness, monkeypatch, "rope_rotate", bad)


def test_mutation_transposed_basis_head(monkeypatch):
    def bad(coef, basis, h, d):
        bh = np.asarray(basis)[h::basis.shape[0] // d][:d]
        return np.asarray(coef) @ bh.T
    _fails(check_projection, monkeypatch, "rebuild_keys", bad)


def test_mutation_residual_not_added(monkeypatch):
    orig = O.reconstruct_chunks

    def bad(sel_bh, coef_b, basis, h, d, chunk, res_idx_bh, res_val_bh, chunk_ptr_bh,
            *rest):
        zero_ptr = np.zeros_like(np.asarray(chunk_ptr_bh))
        return orig(sel_bh, coef_b, basis, h, d, chunk, res_idx_bh, res_val_bh, zero_ptr,
                    *rest)
    _fails(check_full_rank_exactness, monkeypatch, "reconstruct_chunks", bad)


def test_mutation_scores_sum_not_max(monkeypatch):
    _fails(check_landmarks_and_scores, monkeypatch, "chunk_scores",
           lambda qg, lm: (np.asarray(lm) @ np.asarray(qg).T).sum(axis=1))


def test_mutation_topk_ties_to_higher(monkeypatch):
    def bad(scores, k):
        s = np.asarray(scores, np.float64)
        n = s.shape[0]
        order = np.lexsort((-np.arange(n), -s))
        return np.sort(order[:min(k, n)])
    _fails(check_topk, monkeypatch, "topk_ascending", bad)


def test_mutation_predictor_drops_bias(monkeypatch):
    orig = O.predictor
    _fails(check_predictor, monkeypatch, "predictor",
           lambda x, w1, b1, w2, b2, act: orig(x, w1, 0 * np.asarray(b1), w2, b2, act))


def test_mutation_errors_from_rounded_coef(monkeypatch):
    orig = O.residual_errors

    def bad(v_h, coef_exact, *rest):
        return orig(v_h, O.round_to_storage(coef_exact, O.STORE_BF16), *rest)
    _fails(check_residual_pick, monkeypatch, "residual_errors", bad)


def test_mutation_landmark_scaled(monkeypatch):
    orig = O.chunk_landmarks

    def bad(k_cache, chunk):
        return orig(k_cache, chunk) * 1.0001
    _fails(check_landmarks_and_scores, monkeypatch, "chunk_landmarks", bad)


def test_mutation_landmark_of_prerope_keys(monkeypatch):
    """encode averaging the inverse-rotated (pre-RoPE) keys instead of the keys it was
    given: the chunk means differ wherever the rotation angle is non-zero."""
    orig = O.chunk_landmarks
    theta = tiny_shape().theta

    def bad(k_cache, chunk):
        T = k_cache.shape[1]
        k_pre = O.rope_rotate(k_cache, np.arange(T)[None, :, None], theta, inverse=True)
        return orig(k_pre, chunk)
    _fails(check_encode_landmarks, monkeypatch, "chunk_landmarks", bad)


def _range_finder_q(a, omega, n_power):
    a = np.asarray(a, np.float64)
    q = O.cholesky_qr(O.cholesky_qr(a.T @ (a @ omega)))
    for _ in range(n_power):
        q = O.cholesky_qr(O.cholesky_qr(a.T @ (a @ q)))
    return a, q


def test_mutation_basis_without_rayleigh_ritz(monkeypatch):
    def bad(a, rank, omega, n_power=2):
        _, q = _range_finder_q(a, omega, n_power)
        return q[:, :rank]
    _fails(check_fit_basis, monkeypatch, "fit_basis", bad)


def test_mutation_basis_smallest_ritz_vectors(monkeypatch):
    def bad(a, rank, omega, n_power=2):
        a, q = _range_finder_q(a, omega, n_power)
        aq = a @ q
        return q @ np.linalg.eigh(aq.T @ aq)[1][:, :rank]
    _fails(check_fit_basis, monkeypatch, "fit_basis", bad)


def test_mutation_cholesky_qr_wrong_factor(monkeypatch):
    def bad(y):
        y = np.asarray(y, np.float64)
        r_up = np.linalg.cholesky(y.T @ y).T
        return np.linalg.solve(r_up, y.T).T
    _fails(check_cholesky_qr, monkeypatch, "cholesky_qr", bad)


def test_mutation_int4_scale_over_eight(monkeypatch):
    def bad(x):
        x = np.asarray(x, np.float64)
        g = x.reshape(*x.shape[:-1], -1, 32)
        sc = O.f64_to_f16(np.abs(g).max(axis=-1) / 8.0)
        safe = np.where(sc > 0, sc, 1.0)[..., None]
        q = np.where(sc[..., None] > 0, np.clip(np.rint(g / safe), -8, 7), 0.0)
        return q.astype(np.int8).reshape(x.shape), sc
    _fails(check_int4_quantize, monkeypatch, "quantize_int4_g32", bad)


def test_mutation_eviction_keeps_smallest(monkeypatch):
    def bad(lm, n_keep):
        lm = np.asarray(lm, np.float64)
        return O.topk_ascending(-(lm * lm).sum(axis=(0, 2)), n_keep)
    _fails(check_eviction, monkeypatch, "eviction_keep", bad)


def test_mutation_evicted_positions_ignored(monkeypatch):
    """Reconstruction re-applying RoPE at the stored slot instead of the original
    position."""
    orig = O.reconstruct_chunks

    def bad(*args):
        return orig(*args[:15], None)
    _fails(check_evicted_full_rank_exactness, monkeypatch, "reconstruct_chunks", bad)


def test_mutation_suffix_softmax_separate(monkeypatch):
    """Prefix and suffix attended with separate softmaxes, then averaged."""
    def bad(q, cache, basis, w1, b1, w2, b2, ks, vs, *, chunk, top_k, theta, act, sel=None):
        a, sel = O.decode_step(q, cache, basis, w1, b1, w2, b2, chunk=chunk, top_k=top_k,
                               theta=theta, act=act, sel=sel)
        if np.asarray(ks).shape[1] == 0:
            return a, sel
        return 0.5 * (a + O.dense_attention(q, ks, vs)), sel
    _fails(check_suffix_decode, monkeypatch, "decode_step_with_suffix", bad)


def test_mutation_block_indices_not_moved(monkeypatch):
    """The block's residual token indices appended without moving them past the prefix."""
    orig = O.append_block

    def bad(prefix, block, *, prefix_tokens, chunk, block_first_chunk):
        return orig(prefix, block, prefix_tokens=0, chunk=chunk,
                    block_first_chunk=block_first_chunk)
    _fails(check_block_append, monkeypatch, "append_block", bad)


def test_mutation_block_positions_from_zero(monkeypatch):
    """The block compressed as if it started at position 0."""
    orig = O.encode_block

    def bad(*args, first_position, **kw):
        return orig(*args, first_position=0, **kw)
    _fails(check_block_append, monkeypatch, "encode_block", bad)


def test_mutation_block_csr_not_moved(monkeypatch):
    """The block's CSR offsets appended without the prefix's row count."""
    orig = O.append_block

    def bad(prefix, block, **kw):
        out = orig(prefix, block, **kw)
        Np = prefix["landmark"].shape[2]
        out["chunk_ptr"] = np.concatenate([prefix["chunk_ptr"][:, :, :Np], block["chunk_ptr"]],
                                          axis=2)
        return out
    _fails(check_block_append, monkeypatch, "append_block", bad)
