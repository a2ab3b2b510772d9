"""Decode state kept in the context between calls, through the C ABI on the GPU.

The selection kernel keeps its scores in a context buffer that must be back in its reset
state after every call; the attend kernel takes tiles from per-head counters and, inside
lowram_decode_step, waits on per-pair ready flags that the combine kernel clears. These
tests mix entry points and caches on ONE context and compare every result with the
oracle, so a state left over by one call would show up in the next. They also cover the
selection's radix path (k above the fast path's limit) and lowram_landmark_norms."""
import numpy as np
import pytest
import torch

import oracle.lowram_oracle as O
from long_context_decode_02_b200 import synth
from tests import helpers as H
from tests.test_gpu_decode import oracle_decode, prepared

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(cuda_device):
    from long_context_decode_02_b200 import lowram
    return lowram


SMALL = synth.CONFIGS[1].replace(name="state", n_tokens=4096, batch=2, seed=91, n_layers=2)


def _check(L, sh, out, sel, t, co, q):
    sel_np = sel.cpu().numpy()
    osel, scores = O.select_chunks(H.f64(q), co["landmark"], sh.top_k)
    H.compare_selection(sel_np, osel, scores, min(sh.top_k, sh.n_chunks))
    want, _ = oracle_decode(sh, co, t, q, sel=sel_np.astype(np.int64))
    assert H.rel_err(H.f64(out), want) <= H.TOL[sh.dtype]


def test_one_context_mixed_entry_points_and_layers(L, cuda_device):
    sh = SMALL
    dev = cuda_device
    layers = [prepared(sh, layer, dev) for layer in range(2)]
    cfg = L.make_config(sh, decode_variant=L.DECODE_TCGEN05)
    ctx = L.Context(cfg, dev.index or 0)
    ws = torch.empty(L.workspace_size(cfg, L.OP_DECODE), dtype=torch.uint8, device=dev)
    k = min(sh.top_k, sh.n_chunks)
    for step in range(3):
        for layer, (t, t_dev, cdev, co, _) in enumerate(layers):
            params = L.layer_params(*(t_dev[n] for n in ("basis", "w1", "b1", "w2", "b2")))
            q = synth.queries(sh, layer, step)
            qd = q.to(dev)
            out = torch.empty_like(qd)
            sel = torch.full((sh.batch, sh.n_kv_heads, k), -1, dtype=torch.int32, device=dev)
            if (step + layer) % 2 == 0:   # the fused step (selection overlapped with attend)
                L.decode_step(ctx, cdev, params, qd, out, ws, sel_out=sel)
            else:                         # the two sub-steps as separate calls
                L.select_chunks(ctx, cdev["landmark"], cdev["landmark_norm"], qd, sel, ws)
                L.attend_selected(ctx, cdev, params, qd, sel, out, ws)
            assert ctx.last_error() == L.OK
            _check(L, sh, out, sel, t, co, q)
    ctx.close()


def test_selection_radix_path_above_the_fast_limit(L, cuda_device):
    """k = 1100 > 1024: the selection runs the radix select over all scores."""
    sh = SMALL.replace(n_tokens=16384, top_k=1100, batch=1)
    t, t_dev, cdev, co, _ = prepared(sh, 0, cuda_device)
    cfg = L.make_config(sh, decode_variant=L.DECODE_SIMT)
    ctx = L.Context(cfg, cuda_device.index or 0)
    ws = torch.empty(L.workspace_size(cfg, L.OP_DECODE), dtype=torch.uint8, device=cuda_device)
    for step in range(2):
        q = synth.queries(sh, 0, step)
        sel = torch.full((sh.batch, sh.n_kv_heads, sh.top_k), -1, dtype=torch.int32,
                         device=cuda_device)
        L.select_chunks(ctx, cdev["landmark"], cdev["landmark_norm"], q.to(cuda_device), sel, ws)
        assert ctx.last_error() == L.OK
        osel, scores = O.select_chunks(H.f64(q), co["landmark"], sh.top_k)
        H.compare_selection(sel.cpu().numpy(), osel, scores, sh.top_k)
    ctx.close()


def test_landmark_norms_entry_point(L, cuda_device):
    sh = SMALL
    t, t_dev, cdev, co, _ = prepared(sh, 0, cuda_device)
    cfg = L.make_config(sh)
    ctx = L.Context(cfg, cuda_device.index or 0)
    got = torch.full((sh.batch, sh.n_kv_heads), float("nan"), device=cuda_device)
    L.landmark_norms(ctx, cdev["landmark"], got)
    assert ctx.last_error() == L.OK
    g = got.cpu().numpy().astype(np.float64)
    lm = H.f64(cdev["landmark"])
    exact = np.sqrt(np.max(np.sum(lm * lm, axis=-1), axis=-1))
    assert np.all(g >= exact)
    assert np.all(g <= H.landmark_norm_bound(lm).astype(np.float64) * (1 + 2.0 ** -22))
    ctx.close()
