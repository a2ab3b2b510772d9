"""The xKV basis fitted on the GPU (lowram_fit_basis: randomised range finder with
Cholesky-QR, fp64 throughout) against the oracle's fit_basis on the same stored keys and
the same random test matrix (agihunt summary, key paragraph: adjacent layers share one
SVD basis, found by a randomised Cholesky-QR instead of the exact SVD).

The two compute the same quantities in fp64 in different association orders (the GPU
forms A^T A once; the oracle applies A^T (A X)), so the Ritz vectors agree to ~1e-12 and
the stored basis must equal the oracle's rounded to the storage format, column by column
up to each column's sign (the method defines a singular vector only up to sign)."""
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


def group_keys(sh):
    """Stored keys of the two layers of group 0: [B, T, H, d] each (storage dtype)."""
    basis = synth.group_basis(sh, 0)
    ks = []
    for layer in range(2):
        w = synth.layer_weights(sh, layer)
        kb = [synth.layer_kv(sh, basis, w, layer, b)[0] for b in range(sh.batch)]
        ks.append(torch.stack(kb).contiguous())
    return ks


def oracle_rows(sh, ks):
    rows = []
    for k in ks:
        kk = H.f64(k)                                            # [B, T, H, d]
        pos = np.arange(sh.n_tokens)[None, :, None]
        kp = O.rope_rotate(kk, pos, sh.theta, inverse=True)
        rows.append(kp.reshape(-1, sh.kv_dim))
    return np.concatenate(rows)


def check_fit(L, sh, l, n_power, dev, ulps):
    ks = group_keys(sh)
    rng = np.random.default_rng(1234)
    omega = rng.standard_normal((sh.kv_dim, l))
    want = O.fit_basis(oracle_rows(sh, ks), sh.rank, omega, n_power=n_power)
    cfg = L.make_config(sh)
    ctx = L.Context(cfg, dev.index or 0)
    ws = torch.empty(L.fit_basis_workspace_size(cfg, l), dtype=torch.uint8, device=dev)
    out = torch.full((sh.kv_dim, sh.rank), float("nan"), dtype=sh.torch_dtype, device=dev)
    L.fit_basis(ctx, [k.to(dev) for k in ks], torch.from_numpy(omega).to(dev), n_power, out, ws)
    assert ctx.last_error() == L.OK
    ctx.close()
    got = H.f64(out)
    store = O.STORE_BF16 if sh.dtype == "bf16" else O.STORE_F32
    mant = 7 if sh.dtype == "bf16" else 23
    worst = 0.0
    for j in range(sh.rank):
        sgn = 1.0 if got[:, j] @ want[:, j] >= 0 else -1.0
        ref = O.round_to_storage(sgn * want[:, j], store)
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - mant)
        err = np.abs(got[:, j] - ref)
        worst = max(worst, float(np.max(err / ulp)))
        assert np.all(err <= ulps * ulp + 1e-30), (j, float(np.max(err / ulp)))
    # orthonormal columns up to the storage rounding
    assert np.abs(got.T @ got - np.eye(sh.rank)).max() < (2e-2 if sh.dtype == "bf16" else 1e-5)
    print(f"fit_basis {sh.name} l={l} power={n_power}: worst {worst:.2f} ulp")


def test_fit_basis_llama_group(L, cuda_device):
    """D = 1024, rank 160, oversampled test matrix (l = 176), two power steps, bf16."""
    sh = synth.CONFIGS[1].replace(name="fit-b1-t4096", n_tokens=4096, batch=1, seed=61)
    check_fit(L, sh, 176, 2, cuda_device, ulps=1.0)


def test_fit_basis_fp32_small_and_full_width(L, cuda_device):
    """fp32 storage, D = 128, rank 32: an oversampled run, and a full-width test matrix
    with no power step (Rayleigh-Ritz over all of R^D gives the SVD subspace)."""
    sh = synth.CONFIGS[0].replace(name="fit-f32", n_tokens=1024, batch=2, seed=62)
    check_fit(L, sh, 40, 2, cuda_device, ulps=1.0)
    check_fit(L, sh, 128, 0, cuda_device, ulps=1.0)


def test_fit_basis_recovers_the_generating_span(L, cuda_device):
    """Fitted on the synthetic keys (c B_g^T + noise), the basis spans B_g to within the
    key noise: the property the method relies on."""
    sh = synth.CONFIGS[1].replace(name="fit-span", n_tokens=2048, batch=2, seed=63)
    ks = group_keys(sh)
    cfg = L.make_config(sh)
    ctx = L.Context(cfg, cuda_device.index or 0)
    l = sh.rank + 8
    ws = torch.empty(L.fit_basis_workspace_size(cfg, l), dtype=torch.uint8, device=cuda_device)
    omega = torch.randn(sh.kv_dim, l, dtype=torch.float64,
                        generator=torch.Generator().manual_seed(5)).to(cuda_device)
    out = torch.empty(sh.kv_dim, sh.rank, dtype=sh.torch_dtype, device=cuda_device)
    L.fit_basis(ctx, [k.to(cuda_device) for k in ks], omega, 2, out, ws)
    assert ctx.last_error() == L.OK
    ctx.close()
    b = H.f64(out)
    bg = H.f64(synth.group_basis(sh, 0))
    assert np.linalg.norm(b @ b.T - bg @ bg.T, 2) < 0.05
