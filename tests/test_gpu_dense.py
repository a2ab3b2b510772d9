"""The uncompressed baseline (lowram_dense_decode): exact GQA decode attention over the
full bf16 cache, through the C ABI, against the oracle's textbook dense attention
(itself pinned to torch's scaled_dot_product_attention on CPU). The output is exact up
to fp32 accumulation and the final bf16 rounding of out (2^-9 relative), so the bar is
the workload's bf16 tolerance with room to spare."""
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


@pytest.mark.parametrize("over", [
    dict(n_tokens=4096, batch=2),
    dict(n_tokens=1040, batch=3),     # a ragged last split of 16 positions
    dict(n_tokens=32768, batch=1),    # config 1's context
], ids=["t4096b2", "t1040b3", "t32768b1"])
def test_dense_decode_matches_dense_attention(L, cuda_device, over):
    sh = synth.CONFIGS[1].replace(name="dense", seed=31, **over)
    dev = cuda_device
    t = H.stored_layer(sh, 0)
    cfg = L.make_config(sh)
    ctx = L.Context(cfg, dev.index or 0)
    ws = torch.empty(L.workspace_size(cfg, L.OP_DENSE), dtype=torch.uint8, device=dev)
    k, v = t["k"].to(dev), t["v"].to(dev)
    errs = []
    for step in range(2):
        q = synth.queries(sh, 0, step)
        out = torch.full_like(q, float("nan"), device=dev)
        L.dense_decode(ctx, k, v, q.to(dev), out, ws)
        torch.cuda.synchronize()
        want = O.dense_attention(H.f64(q), H.f64(t["k"]), H.f64(t["v"]))
        errs.append(H.rel_err(H.f64(out), want))
    ctx.close()
    print(f"dense decode {over}: max rel err {max(errs):.2e}")
    assert max(errs) <= H.TOL["bf16"]


def test_dense_decode_refuses_unsupported(L, cuda_device):
    sh = synth.CONFIGS[0]                   # fp32, d 64: not the bf16 d-128 kernel
    cfg = L.make_config(sh)
    with pytest.raises(L.LowRAMError) as e:
        L.workspace_size(cfg, L.OP_DENSE)
    assert e.value.status == L.ERR_UNSUPPORTED
