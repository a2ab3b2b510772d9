"""Seeded synthetic workloads shaped like the Llama-3-8B / Mistral-7B GQA caches.

This module only makes inputs. It is shared by the tests, the bench and the smoke check,
and it is the ONLY code both the CPU oracle and the CUDA library see; it holds none of
the method's own steps (no projection, landmark, selection, predictor fit, residual pick
or attention). It builds keys and values with the structure the method exploits, using
torch library calls:

  per 2-layer group g:  basis B_g = Q of the QR of an N(0,1) [D, r] matrix (fp64)
  per layer:            W1 [H, F, d], W2 [H, d, F] Xavier-uniform; b1 = b2 = 0
  per (layer, batch):   c ~ N(0,1) [T, r];  K_pre = c B_g^T + noise * N(0,1)
                        V_h = W2_h act(W1_h K_pre,h) + noise * N(0,1)
                        outliers: floor(outlier_frac * T) tokens per head, drawn without
                        replacement, get N(0, outlier_std^2) added to their whole V row
                        K_cache = K_pre rotated by the token position (RoPE, complex form)
  per (layer, step):    q ~ N(0,1) [B, H_q, d], already rotated

Seeds: ``torch.Generator(device).manual_seed(1000 * config + 97 * layer + 7 * b + s)``
with a distinct small offset ``s`` per stream (documented at each call).
"""
from __future__ import annotations

import dataclasses
import math

import torch
import torch.nn.functional as F

ACT_SILU = 0
ACT_GELU_ERF = 1


@dataclasses.dataclass(frozen=True)
class Shape:
    """All numeric parameters of one workload."""
    name: str
    batch: int
    n_tokens: int
    n_layers: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int
    rank: int
    chunk: int
    top_k: int
    res_frac: float
    mlp_hidden: int
    act: int
    dtype: str            # "bf16" or "f32": storage of every cache/weight/IO tensor
    theta: float
    outlier_frac: float
    steps: int
    noise: float = 0.05
    outlier_std: float = 3.0
    seed: int = 0
    keep_frac: float = 1.0      # fraction of chunks kept by eviction (1: no eviction)
    res_int4: bool = False      # residual rows stored as int4 codes + fp16 scales

    @property
    def n_res(self) -> int:
        """Residual rows per (batch, KV head): a fraction of the tokens the cache holds."""
        return int(math.floor(self.res_frac * self.n_kept_tokens + 1e-9))

    @property
    def n_chunks(self) -> int:
        """Chunks the cache holds (after eviction)."""
        return self.n_kept_chunks

    @property
    def n_kept_chunks(self) -> int:
        return int(math.floor(self.keep_frac * (self.n_tokens // self.chunk) + 1e-9))

    @property
    def n_kept_tokens(self) -> int:
        return self.n_kept_chunks * self.chunk

    @property
    def evicted(self) -> bool:
        return self.n_kept_tokens < self.n_tokens

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def replace(self, **kw) -> "Shape":
        return dataclasses.replace(self, **kw)


# The five workloads. Sizes follow the configuration list of the task; the pages give
# none of them (their models are Llama-3-8B- and Mistral-7B-shaped GQA models).
CONFIGS = {
    0: Shape("tiny-f32-2layer", batch=1, n_tokens=1024, n_layers=2, n_kv_heads=2,
             n_q_heads=8, head_dim=64, rank=32, chunk=8, top_k=16, res_frac=0.125,
             mlp_hidden=128, act=ACT_GELU_ERF, dtype="f32", theta=1e4,
             outlier_frac=0.05, steps=4, seed=0),
    1: Shape("llama8b-layerpair-32k", batch=1, n_tokens=32768, n_layers=2, n_kv_heads=8,
             n_q_heads=32, head_dim=128, rank=160, chunk=8, top_k=256, res_frac=0.2,
             mlp_hidden=256, act=ACT_SILU, dtype="bf16", theta=5e5,
             outlier_frac=0.03, steps=64, seed=1000),
    2: Shape("llama8b-32layer-128k-b8", batch=8, n_tokens=131072, n_layers=32,
             n_kv_heads=8, n_q_heads=32, head_dim=128, rank=160, chunk=8, top_k=256,
             res_frac=0.2, mlp_hidden=256, act=ACT_SILU, dtype="bf16", theta=5e5,
             outlier_frac=0.03, steps=64, seed=2000),
    3: Shape("mistral7b-32layer-262k-b4", batch=4, n_tokens=262144, n_layers=32,
             n_kv_heads=8, n_q_heads=32, head_dim=128, rank=128, chunk=8, top_k=256,
             res_frac=0.15, mlp_hidden=256, act=ACT_SILU, dtype="bf16", theta=1e6,
             outlier_frac=0.03, steps=16, seed=3000),
    # LowRAM-Q/EQ composition: config 2's shapes at 64K, int4 residual rows for the worst
    # 40% of the kept tokens, half the chunks evicted; batch swept 1, 4, 8, 16, 28
    4: Shape("llama8b-32layer-64k-eq", batch=8, n_tokens=65536, n_layers=32, n_kv_heads=8,
             n_q_heads=32, head_dim=128, rank=160, chunk=8, top_k=256, res_frac=0.4,
             mlp_hidden=256, act=ACT_SILU, dtype="bf16", theta=5e5, outlier_frac=0.03,
             steps=16, seed=4000, keep_frac=0.5, res_int4=True),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def group_basis(shape: Shape, group: int, device="cpu") -> torch.Tensor:
    """Orthonormal-column basis [D, r] in fp64 for a 2-layer group (stream offset 1)."""
    g = _gen(device, shape.seed + 97 * 2 * group + 1)
    a = torch.randn(shape.kv_dim, shape.rank, generator=g, device=device,
                    dtype=torch.float64)
    q, _ = torch.linalg.qr(a, mode="reduced")
    return q.contiguous()


def layer_weights(shape: Shape, layer: int, device="cpu"):
    """Per-head predictor weights of one layer, fp64 (stream offset 2).

    Returns w1 [H, F, d], b1 [H, F], w2 [H, d, F], b2 [H, d].
    """
    g = _gen(device, shape.seed + 97 * layer + 2)
    H, Fh, d = shape.n_kv_heads, shape.mlp_hidden, shape.head_dim
    bound = math.sqrt(6.0 / (d + Fh))
    w1 = (torch.rand(H, Fh, d, generator=g, device=device, dtype=torch.float64) * 2 - 1) * bound
    w2 = (torch.rand(H, d, Fh, generator=g, device=device, dtype=torch.float64) * 2 - 1) * bound
    b1 = torch.zeros(H, Fh, device=device, dtype=torch.float64)
    b2 = torch.zeros(H, d, device=device, dtype=torch.float64)
    return w1, b1, w2, b2


def _rotate(x: torch.Tensor, pos: torch.Tensor, theta: float) -> torch.Tensor:
    """Position rotation of the last dim (halves as real/imaginary parts)."""
    d = x.shape[-1]
    freqs = 1.0 / (theta ** (torch.arange(0, d, 2, device=x.device, dtype=torch.float64) / d))
    ang = torch.outer(pos.to(torch.float64), freqs)                       # [T, d/2]
    rot = torch.polar(torch.ones_like(ang), ang)                          # e^{i a}
    z = torch.complex(x[..., : d // 2].to(torch.float64), x[..., d // 2:].to(torch.float64))
    if x.dim() == 3:                                                      # [T, H, d]
        rot = rot[:, None, :]
    z = z * rot
    return torch.cat([z.real, z.imag], dim=-1).to(x.dtype)


def _act(x: torch.Tensor, act: int) -> torch.Tensor:
    return F.silu(x) if act == ACT_SILU else F.gelu(x, approximate="none")


def layer_kv(shape: Shape, basis: torch.Tensor, weights, layer: int, b: int,
             device="cpu", compute_dtype=torch.float64):
    """Keys (post-rotation) and values of one (layer, batch element), [T, H, d] each.

    Stream offset 3. Arithmetic in ``compute_dtype``; returned in the storage dtype.
    """
    g = _gen(device, shape.seed + 97 * layer + 7 * b + 3)
    T, H, d, r = shape.n_tokens, shape.n_kv_heads, shape.head_dim, shape.rank
    bas = basis.to(device=device, dtype=compute_dtype)
    c = torch.randn(T, r, generator=g, device=device, dtype=compute_dtype)
    k_pre = c @ bas.T
    k_pre += shape.noise * torch.randn(T, H * d, generator=g, device=device, dtype=compute_dtype)
    k_pre = k_pre.view(T, H, d)
    w1, b1, w2, b2 = (w.to(device=device, dtype=compute_dtype) for w in weights)
    v = torch.empty(T, H, d, device=device, dtype=compute_dtype)
    for h in range(H):
        hid = _act(F.linear(k_pre[:, h], w1[h], b1[h]), shape.act)
        v[:, h] = F.linear(hid, w2[h], b2[h])
    v += shape.noise * torch.randn(T, H, d, generator=g, device=device, dtype=compute_dtype)
    n_out = int(math.floor(shape.outlier_frac * T + 1e-9))
    if n_out > 0:
        for h in range(H):
            rows = torch.randperm(T, generator=g, device=device)[:n_out]
            v[rows, h] += shape.outlier_std * torch.randn(n_out, d, generator=g,
                                                          device=device, dtype=compute_dtype)
    pos = torch.arange(T, device=device)
    k_cache = _rotate(k_pre, pos, shape.theta)
    st = shape.torch_dtype
    return k_cache.to(st), v.to(st)


def queries(shape: Shape, layer: int, step: int, device="cpu") -> torch.Tensor:
    """q ~ N(0,1) [B, H_q, d] for one (layer, step) in the storage dtype (stream offset 5)."""
    g = _gen(device, shape.seed + 97 * layer + 131 * step + 5)
    q = torch.randn(shape.batch, shape.n_q_heads, shape.head_dim, generator=g,
                    device=device, dtype=torch.float32)
    return q.to(shape.torch_dtype)


def stored(x: torch.Tensor, shape: Shape) -> torch.Tensor:
    """Cast a tensor to the workload's storage dtype."""
    return x.to(shape.torch_dtype)
