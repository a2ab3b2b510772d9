"""tcgen05 building blocks through the C ABI: one 128 x 128 tile product staged with the
exact shared-memory layouts, TMA boxes, swizzles and descriptors of the tensor-core
decode kernel, against an fp64 product of the same bf16 values. Runs first, so a
descriptor problem shows up here before the fused kernel is exercised."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(cuda_device):
    from long_context_decode_02_b200 import lowram
    return lowram


def _tile(L, k, mode, seed, n=128):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(128, k, generator=g).to(torch.bfloat16)
    b = torch.randn(128, k, generator=g).to(torch.bfloat16)
    d = torch.empty(128, 128, dtype=torch.float32, device="cuda")
    L.debug_tc_tile(a.cuda(), b.cuda(), d, k, mode)
    ref = (a.double() @ b.double().T)[:, :n]
    err = (d.double().cpu()[:, :n] - ref).abs().max().item()
    return err, ref.abs().max().item()


@pytest.mark.parametrize("k", [32, 64, 128, 160, 256])
def test_tile_64b_swizzle_gather_layout(L, k):
    err, scale = _tile(L, k, 0, k)
    assert err <= 1e-5 * scale, (err, scale)


def test_tile_128b_swizzle_thread_written_operand(L):
    err, scale = _tile(L, 128, 1, 7)
    assert err <= 1e-5 * scale, (err, scale)


def test_tile_tensor_memory_a_operand(L):
    """A from Tensor Memory (bf16 pairs along K), N = 16: the layout of the weighted
    hidden-activation sum."""
    err, scale = _tile(L, 128, 2, 11, n=16)
    assert err <= 1e-5 * scale, (err, scale)
