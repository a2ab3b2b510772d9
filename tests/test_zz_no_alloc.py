"""The decode entry point that allocates nothing (lowram_decode_step_static), checked
against lowram_decode_step with a caller workspace.

Some callers cannot allocate device memory where they decode. Examples are a serving
loop whose memory pool is fully reserved, a runtime that forbids allocation after
start-up, and a plugin that owns no allocator. lowram_decode_step_static serves them from
a fixed 32 MiB device array inside the library.

This file calls it through the C ABI twice in a row, with different queries. Each call
must match the workspace entry point: the same selected chunks, and outputs within the
bf16 tolerance the other tests use. It also checks that a configuration needing more
scratch than the array holds is refused before anything runs.

The file is named to be collected last, so a failure here stops a `-x` run only after
every other test has run. It needs no state from other tests and runs alone as well.
"""
import numpy as np
import pytest
import torch

from long_context_decode_02_b200 import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def L(cuda_device):
    from long_context_decode_02_b200 import lowram
    return lowram


def test_static_scratch_decode_matches_workspace_decode(L, cuda_device):
    sh = synth.CONFIGS[1].replace(name="no-alloc", n_tokens=4096, batch=2, seed=123)
    dev = cuda_device
    t = H.stored_layer(sh, 0)
    td = {n: x.to(dev) for n, x in t.items()}
    cfg = L.make_config(sh)
    ctx = L.Context(cfg, dev.index or 0)
    cache = L.alloc_cache(cfg, dev)
    params = L.layer_params(*(td[n] for n in ("basis", "w1", "b1", "w2", "b2")))
    enc_ws = torch.empty(L.workspace_size(cfg, L.OP_ENCODE), dtype=torch.uint8, device=dev)
    L.encode(ctx, td["k"], td["v"], params, cache, enc_ws)
    assert ctx.last_error() == L.OK
    dec_ws = torch.empty(L.workspace_size(cfg, L.OP_DECODE), dtype=torch.uint8, device=dev)
    kk = min(sh.top_k, sh.n_chunks)
    queries = [synth.queries(sh, 0, step).to(dev) for step in range(3)]
    refs = []
    for q in queries:
        out_ref = torch.empty_like(q)
        sel_ref = torch.empty(sh.batch, sh.n_kv_heads, kk, dtype=torch.int32, device=dev)
        L.decode_step(ctx, cache, params, q, out_ref, dec_ws, sel_out=sel_ref)
        refs.append((out_ref, sel_ref))
    torch.cuda.synchronize()
    outs = [torch.full_like(q, float("nan")) for q in queries]
    sels = [torch.full_like(refs[0][1], -1) for _ in queries]
    # the first call may load the library's device code (lazy module loading), which
    # reserves the array itself; every later call must take no device memory at all
    L.decode_step_static(ctx, cache, params, queries[0], outs[0], sel_out=sels[0])
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info(dev)
    torch_bytes0 = torch.cuda.memory_allocated(dev)
    # two calls in a row with different queries: the shared array keeps the last call's
    # data; the second one leaves the selection in the array (sel_out = NULL)
    L.decode_step_static(ctx, cache, params, queries[1], outs[1], sel_out=sels[1])
    L.decode_step_static(ctx, cache, params, queries[2], outs[2], sel_out=None)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(dev)[0] == free0
    assert torch.cuda.memory_allocated(dev) == torch_bytes0
    assert ctx.last_error() == L.OK
    for step, (out, sel, (out_ref, sel_ref)) in enumerate(zip(outs, sels, refs)):
        if step < 2:
            assert torch.equal(sel, sel_ref), step
        err = H.rel_err(H.f64(out), H.f64(out_ref))
        assert np.isfinite(err) and err <= TOL_BF16, (step, err)
    ctx.close()


def test_static_scratch_holds_the_128k_batch8_layer():
    """The 32 MiB array covers the decode workspace of a 128K-token, batch-8
    Llama-3-8B-shaped layer (host-only size query; the limit the design notes state)."""
    from long_context_decode_02_b200 import lowram as L
    cfg = L.make_config(synth.CONFIGS[2])
    assert L.workspace_size(cfg, L.OP_DECODE) <= (32 << 20)


def test_static_scratch_refuses_an_oversize_configuration(L, cuda_device):
    big = synth.CONFIGS[2].replace(n_tokens=1 << 20)   # decode workspace far above 32 MiB
    cfg = L.make_config(big)
    assert L.workspace_size(cfg, L.OP_DECODE) > (32 << 20)
    ctx = L.Context(cfg, cuda_device.index or 0)
    st = L.lowram_decode_step_static(ctx.handle, None, None, None, None, None, None)
    assert st == L.ERR_WORKSPACE
    ctx.close()
