"""Plain fp64 CPU oracle for LowRAM's encode and its decode-time hot path.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import or call this module. The library (C-ABI + CUDA kernels)
never calls it, and it shares no code with the library: every function below is written
out from the method's definition, one step per function, with numpy fp64 arithmetic and
library primitives (matmul, sort, cos/sin, erf) only.

Passages followed (the pages print no formula, listing or worked example; each step is
the plainest reading of the prose):

[keys]     "LowRAM: Low-Rank Keys and Amortised Values for Composable KV Cache
           Compression at Test-Time", agihunt.info summary, the paragraph on the key side:
           keys are not predicted; they get xKV cross-layer low-rank compression with
           adjacent layers sharing one SVD basis; RoPE is inverted before compression;
           the prefix is cut into chunks whose mean key is a landmark, and each decode
           step rebuilds only the top-k chunks chosen by the current query.
[values]   same page, the value-cache-amortisation paragraph and the ablation
           paragraph: a lightweight per-head key->value predictor (nonlinear: a linear
           one ablates badly), residuals kept only for the worst-reconstructed tokens,
           chosen by error rather than at random.
[how]      "LowRAM Exploits Key-Value Predictability to Compress the KV Cache"
           (cctest.ai), section "How the method works": bullets "Low-rank keys",
           "Amortised values", "Residuals for difficult tokens", "Selective
           reconstruction".
[abstract] the paper's abstract (zhuanzhiai.com and arxiv.science pages): per-head
           predictor fitted at test time, residuals only for the tokens it
           reconstructs worst, reconstruction of a selected subset of KV pairs at each
           decoding step.
[summary]  the agihunt.info summary, its composition paragraph (quantised residuals,
           eviction) and its limitations paragraph (long generation: the generated
           suffix kept dense and compressed periodically).

Readings taken where the pages are silent (each is listed, with its reason, in the
design notes of the repository):
- RoPE is the rotate-half form: pairs (i, i + d/2), theta_i = theta^(-2i/d), angle
  t * theta_i for token position t = 0..T-1; its inverse is its transpose.
- The xKV basis spans all KV heads of a layer (D = H_kv * d); keys are projected as
  c_t = B^T K_pre,t and rebuilt per head as B_h c_t (B_h = rows h*d .. h*d+d-1).
- The predictor is MLP_h(x) = W2_h act(W1_h x + b1_h) + b2_h applied to the pre-RoPE
  rebuilt key; act is SiLU or erf-GELU.
- Residuals are additive corrections R = V - V_hat for the n_res tokens of largest
  squared error per (batch, kv head), the error taken with the unrounded coefficients,
  ties to the lower token index; the stored residual uses the stored coefficients.
- A chunk's score is the max over the GQA group's query heads of q . landmark; the
  k highest-scoring chunks are selected, ties to the lower chunk index.
- Attention is softmax(q . K_rot / sqrt(d)) over the selected tokens only.
- The group basis, where it is computed rather than given, is the top-r right singular
  subspace of the group's stacked pre-RoPE key rows, found by a randomised range finder
  (subspace iteration, Cholesky-QR applied twice, a Rayleigh-Ritz step) whose random
  test matrix is an input.
- Composition with quantisation (LowRAM-Q): residual rows stored as symmetric int4
  codes with an fp16 scale per 32 elements, s = fp16(max|x| / 7), q = clamp(rne(x / s),
  -8, 7). Composition with eviction (LowRAM-E/EQ): per batch element, the chunks with
  the smallest all-head landmark norm are evicted before compression; the kept chunks
  keep their original RoPE positions.
- Periodic re-compression of the generated suffix: a block of whole chunks is
  compressed like a prefix (same basis and predictor, RoPE inverted at its true
  positions, its own residual budget chosen within the block) and appended after the
  compressed prefix, whose arrays are left as they are.

Every function here is pinned by ``tests/test_oracle_pins.py`` against something other
than itself (closed forms, brute force, invariants, library routines); none is
"parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

ACT_SILU = 0
ACT_GELU_ERF = 1

STORE_F64 = "f64"   # no rounding: used by the exactness pins
STORE_F32 = "f32"
STORE_BF16 = "bf16"


# ----------------------------------------------------------------------------------
# storage precision
# ----------------------------------------------------------------------------------
def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bfloat16 (round to nearest, ties to even); return the bits.

    bfloat16 keeps fp32's sign and 8-bit exponent and the top 7 fraction bits. The
    rounding is done once, from fp64, on the 52-bit fraction: keep 7 bits, round the
    discarded 45 to nearest-even.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    bits = x.view(np.uint64).copy()
    finite = np.isfinite(x)
    drop = np.uint64(45)
    lsb = (bits >> drop) & np.uint64(1)
    bits = np.where(finite, bits + (np.uint64((1 << 44) - 1) + lsb), bits)
    bits &= ~np.uint64((1 << 45) - 1)
    as32 = bits.view(np.float64).astype(np.float32)  # exact: at most 8 significant bits
    return (as32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(u: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits to fp64 exactly."""
    u = np.asarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def round_to_storage(x: np.ndarray, store: str) -> np.ndarray:
    """Value of ``x`` after storing it in the given precision, as fp64."""
    if store == STORE_F64:
        return np.asarray(x, dtype=np.float64).copy()
    if store == STORE_F32:
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    if store == STORE_BF16:
        return bf16_bits_to_f64(f64_to_bf16_bits(x))
    raise ValueError(f"unknown storage precision {store!r}")


# ----------------------------------------------------------------------------------
# RoPE [keys]: inverted before compression, re-applied at reconstruction
# ----------------------------------------------------------------------------------
def rope_inv_freq(d: int, theta: float) -> np.ndarray:
    """theta_i = theta^(-2i/d), i = 0 .. d/2-1 (fp64)."""
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * i / d)


def rope_rotate(x: np.ndarray, pos, theta: float, inverse: bool = False) -> np.ndarray:
    """R(pos) x in the rotate-half form, or R(pos)^T x when ``inverse``.

    x: [..., d]; pos: integer positions broadcastable to x.shape[:-1].
    y_i = x_i cos(a_i) - x_{i+d/2} sin(a_i);  y_{i+d/2} = x_i sin(a_i) + x_{i+d/2} cos(a_i),
    a_i = pos * theta_i. The inverse rotates by -a_i.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_inv_freq(d, theta)
    cs, sn = np.cos(ang), np.sin(ang)
    if inverse:
        sn = -sn
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cs - x2 * sn, x1 * sn + x2 * cs], axis=-1)


# ----------------------------------------------------------------------------------
# cross-layer low-rank keys [keys], [how: Low-rank keys]
# ----------------------------------------------------------------------------------
def project_keys(k_pre_flat: np.ndarray, basis: np.ndarray) -> np.ndarray:
    """c_t = B^T K_pre,t over the flattened D = H_kv*d key of token t.

    k_pre_flat: [..., D]; basis: [D, r] with orthonormal columns -> [..., r].
    """
    return np.asarray(k_pre_flat, dtype=np.float64) @ np.asarray(basis, dtype=np.float64)


def rebuild_keys(coef: np.ndarray, basis: np.ndarray, h: int, d: int) -> np.ndarray:
    """K~_pre,t,h = B_h c_t, B_h = rows h*d .. h*d+d-1 of the basis. -> [..., d]."""
    bh = np.asarray(basis, dtype=np.float64)[h * d:(h + 1) * d, :]
    return np.asarray(coef, dtype=np.float64) @ bh.T


def cholesky_qr(y: np.ndarray) -> np.ndarray:
    """Orthonormal basis of the columns of y (full column rank) by Cholesky-QR: with R
    the upper Cholesky factor of the Gram matrix y^T y (y^T y = R^T R), Q = y R^-1."""
    y = np.asarray(y, dtype=np.float64)
    r_up = np.linalg.cholesky(y.T @ y).T
    return np.linalg.solve(r_up.T, y.T).T


def fit_basis(k_pre_rows: np.ndarray, rank: int, omega: np.ndarray,
              n_power: int = 2) -> np.ndarray:
    """The xKV basis of one layer group from its keys, by a randomised range finder with
    Cholesky-QR in place of an exact SVD ([keys]: adjacent layers share one SVD basis,
    and a randomised Cholesky-QR replaces the exact SVD).

    Reading: the basis is the top-`rank` right singular subspace of A = k_pre_rows (every
    token of every layer of the group as one row of the flattened D = H_kv*d pre-RoPE
    key), found by subspace iteration on A^T A:
      Y = A^T (A omega);  Q = CholQR2(Y);
      n_power times:  Q = CholQR2(A^T (A Q));
      Rayleigh-Ritz:  S = (A Q)^T (A Q), U = its eigenvectors by decreasing eigenvalue;
      basis = Q U[:, :rank]  (orthonormal columns).
    CholQR2 is Cholesky-QR applied twice. omega [D][l], l >= rank, is the random test
    matrix, passed in. Returns [D][rank].
    """
    a = np.asarray(k_pre_rows, dtype=np.float64)
    q = cholesky_qr(cholesky_qr(a.T @ (a @ np.asarray(omega, dtype=np.float64))))
    for _ in range(n_power):
        q = cholesky_qr(cholesky_qr(a.T @ (a @ q)))
    aq = a @ q
    evals, evecs = np.linalg.eigh(aq.T @ aq)
    order = np.argsort(-evals, kind="stable")
    return q @ evecs[:, order[:rank]]


# ----------------------------------------------------------------------------------
# chunk landmarks and top-k chunk selection [keys], [how: Selective reconstruction]
# ----------------------------------------------------------------------------------
def chunk_landmarks(k_cache: np.ndarray, chunk: int) -> np.ndarray:
    """Mean post-RoPE key of every chunk, per KV head.

    k_cache: [B, T, H, d] -> [B, H, T/chunk, d].
    """
    B, T, H, d = k_cache.shape
    assert T % chunk == 0
    grouped = np.asarray(k_cache, dtype=np.float64).reshape(B, T // chunk, chunk, H, d)
    return grouped.mean(axis=2).transpose(0, 2, 1, 3)


def chunk_scores(q_group: np.ndarray, landmark: np.ndarray) -> np.ndarray:
    """Score of each chunk for one KV head: max over the group's query heads of q . L_c.

    q_group: [G, d]; landmark: [N_c, d] -> [N_c].
    """
    dots = np.asarray(landmark, dtype=np.float64) @ np.asarray(q_group, dtype=np.float64).T
    return dots.max(axis=1)


def topk_ascending(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores (ties to the lower index), returned ascending."""
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    k = min(int(k), n)
    order = np.lexsort((np.arange(n), -scores))  # primary: score desc; then index asc
    return np.sort(order[:k]).astype(np.int64)


# ----------------------------------------------------------------------------------
# amortised values [values], [how: Amortised values], [abstract]
# ----------------------------------------------------------------------------------
def activation(x: np.ndarray, act: int) -> np.ndarray:
    """SiLU(x) = x / (1 + e^-x);  GELU(x) = x/2 (1 + erf(x / sqrt 2))."""
    x = np.asarray(x, dtype=np.float64)
    if act == ACT_SILU:
        return x / (1.0 + np.exp(-x))
    if act == ACT_GELU_ERF:
        return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))
    raise ValueError(f"unknown activation {act}")


def predictor(x: np.ndarray, w1, b1, w2, b2, act: int) -> np.ndarray:
    """One head's key->value MLP: V_hat = W2 act(W1 x + b1) + b2.

    x: [..., d]; w1: [F, d]; b1: [F]; w2: [d, F]; b2: [d] -> [..., d].
    """
    hid = activation(np.asarray(x, np.float64) @ np.asarray(w1, np.float64).T
                     + np.asarray(b1, np.float64), act)
    return hid @ np.asarray(w2, np.float64).T + np.asarray(b2, np.float64)


# ----------------------------------------------------------------------------------
# composition with quantisation and eviction ([summary] composition paragraph: residuals
# stored at low precision free memory for more residuals (LowRAM-Q); eviction shortens
# the sequence (LowRAM-E, LowRAM-EQ))
# ----------------------------------------------------------------------------------
INT4_GROUP = 32


def f64_to_f16(x: np.ndarray) -> np.ndarray:
    """Value of ``x`` after rounding to IEEE half precision (nearest, ties to even), as
    fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def quantize_int4_g32(x: np.ndarray):
    """Symmetric int4 codes of a residual row, one fp16 scale per 32 consecutive elements.

    Reading: s = fp16(max|x| / 7) per group; q = clamp(round-half-even(x / s), -8, 7),
    q = 0 where s = 0. x: [..., d] with d % 32 == 0. Returns (codes int8 [..., d],
    scales [..., d/32] as fp64 values of fp16 numbers).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    g = x.reshape(*x.shape[:-1], d // INT4_GROUP, INT4_GROUP)
    s = f64_to_f16(np.abs(g).max(axis=-1) / 7.0)
    safe = np.where(s > 0, s, 1.0)[..., None]
    q = np.where(s[..., None] > 0, np.clip(np.rint(g / safe), -8, 7), 0.0)
    return q.astype(np.int8).reshape(x.shape), s


def dequantize_int4_g32(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """x_hat = q * s, group by group. codes [..., d]; scales [..., d/32] -> [..., d]."""
    codes = np.asarray(codes, dtype=np.float64)
    d = codes.shape[-1]
    g = codes.reshape(*codes.shape[:-1], d // INT4_GROUP, INT4_GROUP)
    return (g * np.asarray(scales, dtype=np.float64)[..., None]).reshape(codes.shape)


def eviction_keep(landmark_b: np.ndarray, n_keep: int) -> np.ndarray:
    """Chunks of one batch element that survive eviction, ascending.

    Reading: the n_keep chunks with the largest all-head landmark norm (the squared L2
    norm over every KV head's landmark, sum_h |L_c,h|^2), ties to the lower chunk index;
    the others are evicted with their coefficients, landmarks and residual rows.
    landmark_b: [H, N_c, d] (the stored landmarks) -> [n_keep].
    """
    lm = np.asarray(landmark_b, dtype=np.float64)
    return topk_ascending((lm * lm).sum(axis=(0, 2)), n_keep)


def encode_evicted(k_cache, v, basis, w1, b1, w2, b2, *, chunk, keep_frac, res_frac, theta,
                   act, store, res_format="store"):
    """Eviction, then compression of what is kept (LowRAM-E / LowRAM-EQ).

    Per batch element: landmarks of the whole prefix (stored rounded), the kept chunks
    (eviction_keep with n_keep = floor(keep_frac * N_c)), then encode() of the kept
    tokens at their original RoPE positions with n_res = floor(res_frac * kept tokens).
    Returns encode()'s cache of the kept tokens plus chunk_pos [B, n_keep], the original
    chunk index of every kept chunk (ascending).
    """
    k_cache = np.asarray(k_cache, np.float64)
    v = np.asarray(v, np.float64)
    B, T, H, d = k_cache.shape
    n_chunks = T // chunk
    n_keep = int(math.floor(keep_frac * n_chunks + 1e-9))
    landmark = round_to_storage(chunk_landmarks(k_cache, chunk), store)
    chunk_pos = np.stack([eviction_keep(landmark[b], n_keep) for b in range(B)])
    rows = (chunk_pos[:, :, None] * chunk + np.arange(chunk)[None, None, :]).reshape(B, -1)
    kk = np.stack([k_cache[b, rows[b]] for b in range(B)])
    vv = np.stack([v[b, rows[b]] for b in range(B)])
    n_res = int(math.floor(res_frac * n_keep * chunk + 1e-9))
    out = encode(kk, vv, basis, w1, b1, w2, b2, chunk=chunk, n_res=n_res, theta=theta,
                 act=act, store=store, positions=rows, res_format=res_format)
    out["chunk_pos"] = chunk_pos
    out["full_landmark"] = landmark
    return out


# ----------------------------------------------------------------------------------
# encode [keys], [values], [how: Residuals for difficult tokens]
# ----------------------------------------------------------------------------------
def residual_errors(v_h: np.ndarray, coef_exact: np.ndarray, basis, h, w1, b1, w2, b2,
                    act) -> np.ndarray:
    """e_t = || V_t,h - MLP_h(B_h c_t) ||^2 with the unrounded coefficients. -> [T]."""
    d = v_h.shape[-1]
    vhat = predictor(rebuild_keys(coef_exact, basis, h, d), w1, b1, w2, b2, act)
    return ((np.asarray(v_h, np.float64) - vhat) ** 2).sum(axis=-1)


def residual_chunk_ptr(res_idx: np.ndarray, n_tokens: int, chunk: int) -> np.ndarray:
    """CSR offsets: residual rows of chunk c are res_idx[ptr[c]:ptr[c+1]]."""
    counts = np.bincount(np.asarray(res_idx) // chunk, minlength=n_tokens // chunk)
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)


def encode(k_cache, v, basis, w1, b1, w2, b2, *, chunk, n_res, theta, act, store,
           positions=None, res_format="store"):
    """Compress one layer's prefix.

    k_cache, v: [B, T, H, d] (post-RoPE keys, values); basis [D, r]; w1 [H, F, d];
    b1 [H, F]; w2 [H, d, F]; b2 [H, d]. ``positions`` [B, T] are the tokens' RoPE
    positions (default 0 .. T-1; after eviction, the kept tokens' original positions).
    ``res_format`` "store" keeps residual rows in the storage precision; "int4" keeps
    them as int4 codes with an fp16 scale per 32 elements (res_q, res_scale), and
    res_val holds their dequantized values. Steps, in the pages' order:
      1. invert RoPE on the keys;
      2. project every token's flattened key onto the shared basis (coefficients are
         stored rounded to ``store``);
      3. landmarks = chunk means of the original post-RoPE keys (stored rounded);
      4. run the per-head predictor on the rebuilt key of every token and take the
         squared error against the true value, with the unrounded coefficients;
      5. per (batch, head) keep the n_res largest-error tokens (ascending indices);
      6. store their residuals V - MLP_h(B_h coef_stored), and the per-chunk CSR.
    """
    k_cache = np.asarray(k_cache, np.float64)
    v = np.asarray(v, np.float64)
    B, T, H, d = k_cache.shape
    D = H * d
    pos = np.broadcast_to(np.arange(T), (B, T)) if positions is None else np.asarray(positions)
    k_pre = rope_rotate(k_cache, pos[:, :, None], theta, inverse=True)
    coef_exact = project_keys(k_pre.reshape(B, T, D), basis)
    coef = round_to_storage(coef_exact, store)
    landmark = round_to_storage(chunk_landmarks(k_cache, chunk), store)
    n_chunks = T // chunk
    err = np.empty((B, H, T))
    res_idx = np.empty((B, H, n_res), np.int64)
    res_val = np.empty((B, H, n_res, d))
    chunk_ptr = np.empty((B, H, n_chunks + 1), np.int64)
    if res_format == "int4":
        res_q = np.empty((B, H, n_res, d), np.int8)
        res_scale = np.empty((B, H, n_res, d // INT4_GROUP))
    for b in range(B):
        for h in range(H):
            err[b, h] = residual_errors(v[b, :, h], coef_exact[b], basis, h,
                                        w1[h], b1[h], w2[h], b2[h], act)
            idx = topk_ascending(err[b, h], n_res)
            vhat_stored = predictor(rebuild_keys(coef[b, idx], basis, h, d),
                                    w1[h], b1[h], w2[h], b2[h], act)
            res_idx[b, h] = idx
            if res_format == "int4":
                codes, scales = quantize_int4_g32(v[b, idx, h] - vhat_stored)
                res_q[b, h], res_scale[b, h] = codes, scales
                res_val[b, h] = dequantize_int4_g32(codes, scales)
            else:
                res_val[b, h] = round_to_storage(v[b, idx, h] - vhat_stored, store)
            chunk_ptr[b, h] = residual_chunk_ptr(idx, T, chunk)
    out = {"coef": coef, "coef_exact": coef_exact, "landmark": landmark,
           "res_idx": res_idx, "res_val": res_val, "chunk_ptr": chunk_ptr, "err": err}
    if res_format == "int4":
        out["res_q"], out["res_scale"] = res_q, res_scale
    return out


# ----------------------------------------------------------------------------------
# periodic re-compression of the generated suffix [summary, limitations paragraph]
# ----------------------------------------------------------------------------------
def encode_block(k_block, v_block, basis, w1, b1, w2, b2, *, chunk, n_res, theta, act,
                 store, first_position, res_format="store"):
    """Compression of a block of whole chunks of generated tokens that sits after the
    compressed prefix: encode() of the block with the same basis and predictor, RoPE
    inverted at the tokens' true positions first_position .. first_position + T_b - 1.

    Reading: the pages name the periodic compression of the generated suffix and leave
    its steps open; the plainest reading keeps every step of encode() and its residual
    budget, applied within the block (n_res of its own largest-error tokens), and leaves
    the compressed prefix as it is (no re-selection of its residuals).
    """
    k_block = np.asarray(k_block, np.float64)
    B, Tb = k_block.shape[:2]
    pos = np.broadcast_to(first_position + np.arange(Tb), (B, Tb))
    return encode(k_block, v_block, basis, w1, b1, w2, b2, chunk=chunk, n_res=n_res,
                  theta=theta, act=act, store=store, positions=pos, res_format=res_format)


def append_block(prefix, block, *, prefix_tokens, chunk, block_first_chunk):
    """The compressed cache of prefix + block: every per-token and per-chunk array of the
    block follows the prefix's (coefficients, landmarks, errors), the block's residual
    rows follow the prefix's rows of each (batch, head) with their token indices moved by
    prefix_tokens, and the block's CSR offsets by the prefix's row count. When either
    part holds chunk positions (eviction), the result holds them for every chunk (the
    prefix's own, or 0 .. N_c-1; the block's chunks at block_first_chunk + i).
    """
    Np = prefix["landmark"].shape[2]
    Nb = block["landmark"].shape[2]
    B = prefix["coef"].shape[0]
    n_res_p = prefix["res_idx"].shape[2]
    out = {
        "coef": np.concatenate([prefix["coef"], block["coef"]], axis=1),
        "coef_exact": np.concatenate([prefix["coef_exact"], block["coef_exact"]], axis=1),
        "landmark": np.concatenate([prefix["landmark"], block["landmark"]], axis=2),
        "err": np.concatenate([prefix["err"], block["err"]], axis=2),
        "res_idx": np.concatenate([prefix["res_idx"], block["res_idx"] + prefix_tokens], axis=2),
        "res_val": np.concatenate([prefix["res_val"], block["res_val"]], axis=2),
        "chunk_ptr": np.concatenate([prefix["chunk_ptr"][:, :, :Np],
                                     block["chunk_ptr"] + n_res_p], axis=2),
    }
    for key in ("res_q", "res_scale"):
        if key in prefix:
            out[key] = np.concatenate([prefix[key], block[key]], axis=2)
    if prefix.get("chunk_pos") is not None or block_first_chunk != Np:
        pp = prefix.get("chunk_pos")
        pp = np.broadcast_to(np.arange(Np), (B, Np)) if pp is None else np.asarray(pp)
        out["chunk_pos"] = np.concatenate(
            [pp, np.broadcast_to(block_first_chunk + np.arange(Nb), (B, Nb))], axis=1)
    return out


# ----------------------------------------------------------------------------------
# decode step [keys], [how: Selective reconstruction], [abstract]
# ----------------------------------------------------------------------------------
def select_chunks(q, landmark, top_k):
    """Per (batch, KV head): the top_k chunks by landmark score, ascending.

    q: [B, H_q, d]; landmark: [B, H, N_c, d] -> (sel [B, H, k], scores [B, H, N_c]).
    """
    q = np.asarray(q, np.float64)
    B, Hq, d = q.shape
    H, n_chunks = landmark.shape[1], landmark.shape[2]
    G = Hq // H
    k = min(int(top_k), n_chunks)
    sel = np.empty((B, H, k), np.int64)
    scores = np.empty((B, H, n_chunks))
    for b in range(B):
        for h in range(H):
            scores[b, h] = chunk_scores(q[b, h * G:(h + 1) * G], landmark[b, h])
            sel[b, h] = topk_ascending(scores[b, h], k)
    return sel, scores


def reconstruct_chunks(sel_bh, coef_b, basis, h, d, chunk, res_idx_bh, res_val_bh,
                       chunk_ptr_bh, w1, b1, w2, b2, act, theta, chunk_pos_b=None):
    """Rebuild K (post-RoPE) and V for the selected chunks of one (batch, KV head).

    Returns (tokens [n], k_rot [n, d], v_rec [n, d]) with tokens (rows of the cache) in
    selection order. V = MLP_h(B_h coef_t), plus the stored residual R_t where t holds
    one. ``chunk_pos_b`` maps a stored chunk to its original chunk index (eviction): RoPE
    is re-applied at the original positions.
    """
    sel_bh = np.asarray(sel_bh, np.int64)
    tokens = (sel_bh[:, None] * chunk + np.arange(chunk)[None, :]).reshape(-1)
    base = sel_bh if chunk_pos_b is None else np.asarray(chunk_pos_b, np.int64)[sel_bh]
    positions = (base[:, None] * chunk + np.arange(chunk)[None, :]).reshape(-1)
    k_pre = rebuild_keys(np.asarray(coef_b, np.float64)[tokens], basis, h, d)
    k_rot = rope_rotate(k_pre, positions, theta)
    v_rec = predictor(k_pre, w1, b1, w2, b2, act)
    for slot, c in enumerate(sel_bh):
        for i in range(int(chunk_ptr_bh[c]), int(chunk_ptr_bh[c + 1])):
            t = int(res_idx_bh[i])
            assert c * chunk <= t < (c + 1) * chunk, "residual index outside its chunk"
            v_rec[slot * chunk + (t - c * chunk)] += res_val_bh[i]
    return tokens, k_rot, v_rec


def decode_step(q, cache, basis, w1, b1, w2, b2, *, chunk, top_k, theta, act, sel=None):
    """One decode step of one layer over the compressed cache.

    q: [B, H_q, d] (post-RoPE). cache: dict with coef [B,T,r], landmark [B,H,N_c,d],
    res_idx [B,H,n_res], res_val [B,H,n_res,d], chunk_ptr [B,H,N_c+1], and after eviction
    chunk_pos [B,N_c] (original chunk index of each stored chunk). ``sel`` may override
    the selection (used when a caller's selection differs only by ties).
    Returns (out [B, H_q, d], sel [B, H, k]).
    """
    q = np.asarray(q, np.float64)
    B, Hq, d = q.shape
    H = cache["landmark"].shape[1]
    G = Hq // H
    if sel is None:
        sel, _ = select_chunks(q, cache["landmark"], top_k)
    out = np.empty((B, Hq, d))
    for b in range(B):
        for h in range(H):
            _, k_rot, v_rec = reconstruct_chunks(
                sel[b, h], cache["coef"][b], basis, h, d, chunk,
                cache["res_idx"][b, h], cache["res_val"][b, h], cache["chunk_ptr"][b, h],
                w1[h], b1[h], w2[h], b2[h], act, theta,
                None if cache.get("chunk_pos") is None else cache["chunk_pos"][b])
            for g in range(G):
                z = k_rot @ q[b, h * G + g] / math.sqrt(d)
                p = np.exp(z - z.max())
                p /= p.sum()
                out[b, h * G + g] = p @ v_rec
    return out, np.asarray(sel)


def decode_step_with_suffix(q, cache, basis, w1, b1, w2, b2, k_suffix, v_suffix, *, chunk,
                            top_k, theta, act, sel=None):
    """One decode step over the compressed prefix plus an uncompressed suffix of
    generated tokens (the pages leave long generation to a suffix that is compressed
    periodically, agihunt summary, limitations paragraph).

    Reading: one softmax over the union of the selected chunks' rebuilt tokens and every
    suffix token; the suffix keys arrive post-RoPE like the cache's original keys.
    k_suffix, v_suffix: [B, S, H, d] (S may be 0). Returns (out [B, H_q, d], sel).
    """
    q = np.asarray(q, np.float64)
    ks, vs = np.asarray(k_suffix, np.float64), np.asarray(v_suffix, np.float64)
    B, Hq, d = q.shape
    H = cache["landmark"].shape[1]
    G = Hq // H
    if sel is None:
        sel, _ = select_chunks(q, cache["landmark"], top_k)
    out = np.empty((B, Hq, d))
    for b in range(B):
        for h in range(H):
            _, k_rot, v_rec = reconstruct_chunks(
                sel[b, h], cache["coef"][b], basis, h, d, chunk,
                cache["res_idx"][b, h], cache["res_val"][b, h], cache["chunk_ptr"][b, h],
                w1[h], b1[h], w2[h], b2[h], act, theta,
                None if cache.get("chunk_pos") is None else cache["chunk_pos"][b])
            keys = np.concatenate([k_rot, ks[b, :, h]])
            vals = np.concatenate([v_rec, vs[b, :, h]])
            for g in range(G):
                z = keys @ q[b, h * G + g] / math.sqrt(d)
                p = np.exp(z - z.max())
                p /= p.sum()
                out[b, h * G + g] = p @ vals
    return out, np.asarray(sel)


def dense_attention(q, k_cache, v):
    """Textbook GQA decode attention over the full uncompressed cache.

    q: [B, H_q, d]; k_cache, v: [B, T, H, d] -> [B, H_q, d].
    """
    q = np.asarray(q, np.float64)
    k_cache = np.asarray(k_cache, np.float64)
    v = np.asarray(v, np.float64)
    B, Hq, d = q.shape
    H = k_cache.shape[2]
    G = Hq // H
    out = np.empty((B, Hq, d))
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            z = k_cache[b, :, h, :] @ q[b, hq] / math.sqrt(d)
            p = np.exp(z - z.max())
            p /= p.sum()
            out[b, hq] = p @ v[b, :, h, :]
    return out
