"""CPU checks of the C-ABI library: it builds, loads, exports every symbol include/lowram.h
declares, and its host-side validation, layouts and status strings behave (no kernel is
launched; no GPU is needed)."""
import ctypes
import re

import pytest


@pytest.fixture(scope="module")
def L():
    from long_context_decode_02_b200 import build
    build.build()
    from long_context_decode_02_b200 import lowram
    return lowram


def _declared(header_path):
    text = open(header_path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lowram_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = _declared(L.HEADER_PATH)
    assert len(names) >= 10
    lib = ctypes.CDLL(L.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared but not exported"
    assert set(names) == set(L.EXPORTED)


def _cfg(L, **kw):
    from long_context_decode_02_b200 import synth
    return L.make_config(synth.CONFIGS[1], **kw)


def test_check_config(L):
    from long_context_decode_02_b200 import synth
    for i, sh in synth.CONFIGS.items():
        c = L.make_config(sh)
        assert L.lowram_check_config(ctypes.byref(c)) == L.OK, i
    bad = [
        (dict(n_q_heads=30), L.ERR_SHAPE),            # H_q % H_kv
        (dict(n_tokens=32770), L.ERR_SHAPE),          # T % C
        (dict(top_k=0), L.ERR_SHAPE),
        (dict(n_res=-1), L.ERR_SHAPE),
        (dict(n_res=32769), L.ERR_SHAPE),
        (dict(head_dim=96), L.ERR_UNSUPPORTED),
        (dict(rank=24), L.ERR_UNSUPPORTED),
        (dict(mlp_hidden=192), L.ERR_UNSUPPORTED),
        (dict(chunk=3, n_tokens=32769), L.ERR_UNSUPPORTED),
        (dict(act=7), L.ERR_INVALID_ARG),
        (dict(dtype=5), L.ERR_INVALID_ARG),
        (dict(reserved=1), L.ERR_INVALID_ARG),
        (dict(rope_theta=-1.0), L.ERR_INVALID_ARG),
        (dict(dtype=L.DTYPE_F32, decode_variant=L.DECODE_TCGEN05), L.ERR_UNSUPPORTED),
        (dict(rank=192, decode_variant=L.DECODE_TCGEN05), L.ERR_UNSUPPORTED),
        (dict(res_format=2), L.ERR_INVALID_ARG),
        (dict(n_positions=-8), L.ERR_SHAPE),
        (dict(n_positions=16384), L.ERR_SHAPE),      # fewer positions than stored tokens
        (dict(n_positions=65540), L.ERR_SHAPE),      # not a multiple of the chunk
        (dict(res_format=1, rank=192), L.ERR_UNSUPPORTED),   # int4 needs the tc encode
        (dict(res_format=1, dtype=L.DTYPE_F32), L.ERR_UNSUPPORTED),
    ]
    for over, want in bad:
        c = _cfg(L, **over)
        assert L.lowram_check_config(ctypes.byref(c)) == want, over
    assert L.lowram_check_config(None) == L.ERR_INVALID_ARG


def test_cache_layout_and_workspace(L):
    c = _cfg(L)
    sizes = L.cache_layout(c)
    B, T, H, d, r = 1, 32768, 8, 128, 160
    n_res = int(0.2 * T)
    assert sizes == [B * T * r * 2, B * H * (T // 8) * d * 2, B * H * n_res * 4,
                     B * H * n_res * d * 2, B * H * (T // 8 + 1) * 4, B * H * 4, 0, 0]
    for op in (L.OP_ENCODE, L.OP_DECODE, L.OP_DENSE):
        assert L.workspace_size(c, op) > 0
    with pytest.raises(L.LowRAMError):          # eviction needs n_positions > n_tokens
        L.workspace_size(c, L.OP_EVICT)
    # LowRAM-EQ: half the chunks kept, int4 residual rows with fp16 scales per 32
    from long_context_decode_02_b200 import synth
    sh = synth.CONFIGS[4]
    ce = L.make_config(sh)
    assert ce.n_tokens == sh.n_tokens // 2 and ce.n_positions == sh.n_tokens
    assert ce.res_format == L.RES_INT4_G32
    Be, Te, nre = sh.batch, ce.n_tokens, ce.n_res
    assert nre == int(0.4 * Te)
    se = L.cache_layout(ce)
    assert se[3] == Be * H * nre * d // 2                 # two codes per byte
    assert se[6] == Be * (Te // 8) * 4                    # chunk_pos
    assert se[7] == Be * H * nre * (d // 32) * 2          # fp16 scales
    assert L.workspace_size(ce, L.OP_EVICT) >= Be * (sh.n_tokens // 8) * 9
    n = ctypes.c_size_t()
    assert L.lowram_workspace_size(ctypes.byref(c), 9, ctypes.byref(n)) == L.ERR_INVALID_ARG


def test_status_strings(L):
    for s in range(0, 9):
        assert L.lowram_status_string(s)
    assert b"unknown" in L.lowram_status_string(99)


def test_calls_validate_before_any_launch(L):
    cs = L.lowram_cache()
    ps = L.lowram_layer_params()
    assert L.lowram_decode_step(None, ctypes.byref(cs), ctypes.byref(ps), None, None, None, None,
                                0, None) == L.ERR_INVALID_ARG
    assert L.lowram_encode(None, None, None, ctypes.byref(ps), ctypes.byref(cs), None, 0,
                           None) == L.ERR_INVALID_ARG
    assert L.lowram_last_error(None) == L.ERR_INVALID_ARG
    L.lowram_destroy(None)
    # misaligned pointers are refused on the host
    assert L.lowram_debug_tc_tile(ctypes.c_void_p(16), ctypes.c_void_p(17), ctypes.c_void_p(32),
                                  64, 0, None) == L.ERR_ALIGN
    assert L.lowram_debug_tc_tile(ctypes.c_void_p(16), ctypes.c_void_p(32), ctypes.c_void_p(48),
                                  48, 0, None) == L.ERR_UNSUPPORTED


def test_create_without_device_fails_cleanly(L):
    import torch
    c = _cfg(L)
    h = ctypes.c_void_p()
    dev = 10_000 if torch.cuda.is_available() else 0
    st = L.lowram_create(ctypes.byref(c), dev, ctypes.byref(h))
    assert st == L.ERR_CUDA and not h.value
