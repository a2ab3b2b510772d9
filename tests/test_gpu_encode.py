"""Encode parity through the C ABI: GPU lowram_encode against the oracle's encode on the
same stored keys, values, basis and weights.

Bar: residual token indices bit-exact except ties within 1e-5 of the k-th error
(reported); chunk CSR identical where the indices are; coefficients and landmarks
within one storage rounding; residual rows within the decode tolerance. End-to-end
(GPU encode -> GPU decode vs oracle encode -> oracle decode) checks outputs only."""
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


def gpu_encode(L, shape, t, device):
    cfg = L.make_config(shape)
    ctx = L.Context(cfg, device.index or 0)
    cache = L.alloc_cache(cfg, device)
    td = {k: v.to(device) for k, v in t.items()}
    params = L.layer_params(*(td[n] for n in ("basis", "w1", "b1", "w2", "b2")))
    ws = torch.empty(L.workspace_size(cfg, L.OP_ENCODE), dtype=torch.uint8, device=device)
    L.encode(ctx, td["k"], td["v"], params, cache, ws)
    st = ctx.last_error()
    assert st == L.OK, L.lowram_status_string(st)
    return ctx, cfg, cache, td, params


def ulp_bound(x, dtype):
    """One unit in the last place of the storage format at |x|."""
    mant = 7 if dtype == "bf16" else 23
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-30)))
    return 2.0 ** (e - mant)


def check_encode(L, shape, device):
    t = H.stored_layer(shape, 0)
    enc = H.oracle_encode(shape, t)
    ctx, cfg, cache, td, params = gpu_encode(L, shape, t, device)
    got_idx = cache["res_idx"].cpu().numpy()
    ties = H.compare_selection(got_idx, enc["res_idx"], enc["err"], shape.n_res)
    same = np.all(got_idx == enc["res_idx"], axis=-1)
    ptr = cache["chunk_ptr"].cpu().numpy()
    assert np.array_equal(ptr[same], enc["chunk_ptr"][same])
    for b in range(shape.batch):
        for h in range(shape.n_kv_heads):
            cnt = np.bincount(got_idx[b, h] // shape.chunk, minlength=shape.n_chunks)
            assert np.array_equal(np.diff(ptr[b, h]), cnt)
    # coefficients and landmarks: the GPU's fp32 value rounds to the same storage value,
    # or to a neighbour when the exact value lies within fp32 error of a rounding midpoint
    for name in ("coef", "landmark"):
        g, w = H.f64(cache[name]), enc[name]
        bound = ulp_bound(w, shape.dtype) * 1.01 + 1e-6 * np.abs(w).max()
        if name == "coef" and shape.dtype == "f32":
            # fp32 storage is no coarser than the fp32 arithmetic, so one storage rounding
            # does not cover it: add the bound of an fp32 dot product of n = H d terms
            # (RoPE inversion included as a few more), gamma_n sum_i |k_i B_i|
            kpre = O.rope_rotate(H.f64(t["k"]), np.arange(shape.n_tokens)[None, :, None],
                                 shape.theta, inverse=True)
            kpre = kpre.reshape(shape.batch, shape.n_tokens, -1)
            n = kpre.shape[-1] + 8
            u = 2.0 ** -24
            bound = bound + (n * u / (1 - n * u)) * (np.abs(kpre) @ np.abs(H.f64(t["basis"])))
        assert np.all(np.abs(g - w) <= bound), (name, float(np.max(np.abs(g - w) - bound)))
    # landmark_norm: an upper bound of max_c |L_c|_2 of the stored landmarks, within two
    # fp32 steps of the definition written out on the host
    got_n = cache["landmark_norm"].cpu().numpy().astype(np.float64)
    lm = H.f64(cache["landmark"])
    exact = np.sqrt(np.max(np.sum(lm * lm, axis=-1), axis=-1))
    assert np.all(got_n >= exact)
    assert np.all(got_n <= H.landmark_norm_bound(lm).astype(np.float64) * (1 + 2.0 ** -22))
    # residual rows: R = V - MLP_h(B_h coef_stored) against the coefficients this side
    # stored (which may differ from the oracle's by one rounding), exact in fp64, then
    # compared with the stored row within one rounding step
    p = H.oracle_params(t)
    gcoef, gval = H.f64(cache["coef"]), H.f64(cache["res_val"])
    v64 = H.f64(t["v"])
    d = shape.head_dim
    for b in range(shape.batch):
        for h in range(shape.n_kv_heads):
            idx = got_idx[b, h]
            if idx.size == 0:
                continue
            want = v64[b, idx, h] - O.predictor(O.rebuild_keys(gcoef[b, idx], p["basis"], h, d),
                                                p["w1"][h], p["b1"][h], p["w2"][h], p["b2"][h],
                                                shape.act)
            bound = 2 * ulp_bound(want, shape.dtype) + 1e-5 * np.abs(want).max()
            err = np.abs(gval[b, h] - want)
            assert np.all(err <= bound), ("res_val", b, h, float(np.max(err - bound)))
    return ties, ctx, cfg, cache, td, params, t, enc


def test_config0_encode(L, cuda_device):
    sh = synth.CONFIGS[0]
    ties, *_ = check_encode(L, sh, cuda_device)
    H.assert_ties_bounded(ties, sh.batch * sh.n_kv_heads, "config0 residual pick")


def test_config1_encode(L, cuda_device):
    sh = synth.CONFIGS[1]
    ties, *_ = check_encode(L, sh, cuda_device)
    H.assert_ties_bounded(ties, sh.batch * sh.n_kv_heads, "config1 residual pick")


@pytest.mark.parametrize("cfg_id", [0, 1])
def test_end_to_end(L, cuda_device, cfg_id):
    sh = synth.CONFIGS[cfg_id]
    ties, ctx, cfg, cache, td, params, t, enc = check_encode(L, sh, cuda_device)
    p = H.oracle_params(t)
    for step in range(2):
        q = synth.queries(sh, 0, step)
        out = torch.empty_like(q, device=cuda_device)
        ws = torch.empty(L.workspace_size(cfg, L.OP_DECODE), dtype=torch.uint8,
                         device=cuda_device)
        L.decode_step(ctx, cache, params, q.to(cuda_device), out, ws)
        assert ctx.last_error() == L.OK
        want, _ = O.decode_step(H.f64(q), enc, p["basis"], p["w1"], p["b1"], p["w2"], p["b2"],
                                chunk=sh.chunk, top_k=sh.top_k, theta=sh.theta, act=sh.act)
        err = H.rel_err(H.f64(out), want)
        assert err <= H.TOL[sh.dtype], err


def test_encode_edge_budgets(L, cuda_device):
    for over in (dict(res_frac=0.0), dict(res_frac=1.0), dict(res_frac=1.0 / 1024)):
        sh = synth.CONFIGS[0].replace(n_tokens=1024, **over)
        check_encode(L, sh, cuda_device)


@pytest.mark.parametrize("over", [
    dict(res_frac=0.0),                       # no residual rows: no residual-row pass
    dict(res_frac=1.0),                       # every token picked
    dict(res_frac=1.0 / 1024),                # two rows per (b, h)
    dict(res_frac=0.3),                       # 614 rows: a ragged last tile of 128
    dict(rank=128, act=synth.ACT_GELU_ERF),   # the other activation and rank
    dict(rank=32, batch=3),
], ids=["nores", "allres", "tworows", "ragged", "r128gelu", "r32b3"])
def test_tensor_core_encode_edges(L, cuda_device, over):
    """bf16, d 128, F 256: the tensor-core encode (projection and predictor on tcgen05)
    against the oracle, with the same bars as above."""
    kw = dict(name="enc-tc", n_tokens=2048, batch=2, seed=55)
    kw.update(over)
    sh = synth.CONFIGS[1].replace(**kw)
    ties, *_ = check_encode(L, sh, cuda_device)
    H.assert_ties_bounded(ties, sh.batch * sh.n_kv_heads, f"tc encode {over}")


@pytest.mark.parametrize("rank", [160, 256], ids=["r160", "r256"])
def test_f32_d128_encode(L, cuda_device, rank):
    """fp32 storage at d 128, F 256: the CUDA-core projection and the fp64 re-score with
    its largest staged operands (W1_h^T in fp32 is 128 KB; at r 256 so is a head's basis
    block) against the oracle, with the same bars as above."""
    sh = synth.CONFIGS[1].replace(name="enc-f32-d128", dtype="f32", n_tokens=2048, batch=1,
                                  rank=rank, seed=77)
    ties, *_ = check_encode(L, sh, cuda_device)
    H.assert_ties_bounded(ties, sh.batch * sh.n_kv_heads, f"f32 d128 encode r{rank}")
