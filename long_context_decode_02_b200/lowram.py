"""ctypes binding of liblowram.so (include/lowram.h). Argument marshalling only: every
step of encode and decode runs in the library's CUDA kernels.

Importing this module loads the library and raises if it is missing; there is no
fallback path. Build it with ``python -m long_context_decode_02_b200.build``.

Functions with the C names take raw integers/pointers; the helpers below them take
torch tensors (device memory and streams only).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblowram.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "lowram.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m long_context_decode_02_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

# status codes
OK = 0
ERR_INVALID_ARG = 1
ERR_SHAPE = 2
ERR_ALIGN = 3
ERR_UNSUPPORTED = 4
ERR_WORKSPACE = 5
ERR_CUDA = 6
ERR_DEVICE_CHECK = 7
ERR_TIMEOUT = 8

DTYPE_F32 = 0
DTYPE_BF16 = 1
ACT_SILU = 0
ACT_GELU_ERF = 1
DECODE_AUTO = 0
DECODE_SIMT = 1
DECODE_TCGEN05 = 2
OP_ENCODE = 0
OP_DECODE = 1
OP_DENSE = 2
OP_EVICT = 3
RES_STORE = 0
RES_INT4_G32 = 1


class lowram_config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_tokens", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("mlp_hidden", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("n_res", ctypes.c_int32),
                ("act", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("decode_variant", ctypes.c_int32), ("res_format", ctypes.c_int32),
                ("n_positions", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("rope_theta", ctypes.c_double)]


class lowram_layer_params(ctypes.Structure):
    _fields_ = [("basis", ctypes.c_void_p), ("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("b2", ctypes.c_void_p)]


class lowram_cache(ctypes.Structure):
    _fields_ = [("coef", ctypes.c_void_p), ("landmark", ctypes.c_void_p),
                ("res_idx", ctypes.c_void_p), ("res_val", ctypes.c_void_p),
                ("chunk_ptr", ctypes.c_void_p), ("landmark_norm", ctypes.c_void_p),
                ("chunk_pos", ctypes.c_void_p), ("res_scale", ctypes.c_void_p)]


_P = ctypes.c_void_p
_S = ctypes.c_int
_sig = {
    "lowram_check_config": (_S, [ctypes.POINTER(lowram_config)]),
    "lowram_create": (_S, [ctypes.POINTER(lowram_config), ctypes.c_int, ctypes.POINTER(_P)]),
    "lowram_destroy": (None, [_P]),
    "lowram_cache_layout": (_S, [ctypes.POINTER(lowram_config), ctypes.POINTER(ctypes.c_size_t)]),
    "lowram_workspace_size": (_S, [ctypes.POINTER(lowram_config), ctypes.c_int,
                                   ctypes.POINTER(ctypes.c_size_t)]),
    "lowram_encode": (_S, [_P, _P, _P, ctypes.POINTER(lowram_layer_params),
                           ctypes.POINTER(lowram_cache), _P, ctypes.c_size_t, _P]),
    "lowram_decode_step": (_S, [_P, ctypes.POINTER(lowram_cache),
                                ctypes.POINTER(lowram_layer_params), _P, _P, _P, _P,
                                ctypes.c_size_t, _P]),
    "lowram_select_chunks": (_S, [_P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "lowram_landmark_norms": (_S, [_P, _P, _P, _P]),
    "lowram_attend_selected": (_S, [_P, ctypes.POINTER(lowram_cache),
                                    ctypes.POINTER(lowram_layer_params), _P, _P, _P, _P,
                                    ctypes.c_size_t, _P]),
    "lowram_decode_step_static": (_S, [_P, ctypes.POINTER(lowram_cache),
                                       ctypes.POINTER(lowram_layer_params), _P, _P, _P, _P]),
    "lowram_last_error": (_S, [_P]),
    "lowram_status_string": (ctypes.c_char_p, [_S]),
    "lowram_debug_tc_tile": (_S, [_P, _P, _P, ctypes.c_int32, ctypes.c_int32, _P]),
    "lowram_dense_decode": (_S, [_P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "lowram_evict": (_S, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "lowram_append": (_S, [_P, ctypes.POINTER(lowram_cache), _P, ctypes.POINTER(lowram_cache),
                           _P, ctypes.POINTER(lowram_cache), _P]),
    "lowram_decode_step_suffix": (_S, [_P, ctypes.POINTER(lowram_cache),
                                       ctypes.POINTER(lowram_layer_params), _P, _P, _P,
                                       ctypes.c_int32, ctypes.c_int32, _P, _P, _P,
                                       ctypes.c_size_t, _P]),
    "lowram_suffix_workspace_size": (_S, [ctypes.POINTER(lowram_config), ctypes.c_int32,
                                          ctypes.POINTER(ctypes.c_size_t)]),
    "lowram_fit_basis": (_S, [_P, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32, _P,
                              ctypes.c_int32, ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]),
    "lowram_fit_basis_workspace_size": (_S, [ctypes.POINTER(lowram_config), ctypes.c_int32,
                                             ctypes.POINTER(ctypes.c_size_t)]),
    "lowram_debug_reconstruct": (_S, [_P, ctypes.POINTER(lowram_cache),
                                      ctypes.POINTER(lowram_layer_params), _P, _P, _P, _P, _P,
                                      _P, _P, ctypes.c_size_t, _P]),
    "lowram_debug_attend_unpublished": (_S, [_P, ctypes.POINTER(lowram_cache),
                                             ctypes.POINTER(lowram_layer_params), _P, _P, _P,
                                             _P, ctypes.c_size_t, _P]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args
    globals()[_name] = _f
EXPORTED = tuple(_sig)


class LowRAMError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lowram_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def check(status: int, where: str) -> None:
    if status != OK:
        raise LowRAMError(status, where)


# ------------------------------------------------------------------ torch helpers
def make_config(shape, decode_variant: int = DECODE_AUTO, **over) -> lowram_config:
    """lowram_config from a workload shape (long_context_decode_02_b200.synth.Shape)."""
    kept = getattr(shape, "n_kept_tokens", shape.n_tokens)
    c = lowram_config(batch=shape.batch, n_tokens=kept, n_kv_heads=shape.n_kv_heads,
                      n_q_heads=shape.n_q_heads, head_dim=shape.head_dim, rank=shape.rank,
                      chunk=shape.chunk, mlp_hidden=shape.mlp_hidden, top_k=shape.top_k,
                      n_res=shape.n_res, act=shape.act,
                      dtype=DTYPE_BF16 if shape.dtype == "bf16" else DTYPE_F32,
                      decode_variant=decode_variant,
                      res_format=RES_INT4_G32 if getattr(shape, "res_int4", False) else RES_STORE,
                      n_positions=shape.n_tokens if kept < shape.n_tokens else 0,
                      reserved=0, rope_theta=shape.theta)
    for k, v in over.items():
        setattr(c, k, v)
    return c


def _ptr(t):
    """Device address of a dense row-major tensor (strided views are refused: the C ABI
    takes plain pointers and reads every array densely)."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError(f"tensor of shape {tuple(t.shape)} is not contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def cache_layout(cfg: lowram_config):
    out = (ctypes.c_size_t * 8)()
    check(lowram_cache_layout(ctypes.byref(cfg), out), "lowram_cache_layout")
    return list(out)


def workspace_size(cfg: lowram_config, op: int) -> int:
    n = ctypes.c_size_t()
    check(lowram_workspace_size(ctypes.byref(cfg), op, ctypes.byref(n)), "lowram_workspace_size")
    return n.value


class Context:
    """Owns a lowram_ctx (RoPE tables, status word, counters) on one device."""

    def __init__(self, cfg: lowram_config, device: int = 0):
        self.cfg = cfg
        self._h = ctypes.c_void_p()
        check(lowram_create(ctypes.byref(cfg), device, ctypes.byref(self._h)), "lowram_create")

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h:
            lowram_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def last_error(self) -> int:
        return lowram_last_error(self._h)


def layer_params(basis, w1, b1, w2, b2) -> lowram_layer_params:
    """Parameter block of one layer. It keeps references to the tensors, so their device
    memory stays allocated while the block is in use."""
    p = lowram_layer_params(_ptr(basis), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2))
    p._refs = (basis, w1, b1, w2, b2)
    return p


def cache_struct(coef, landmark, res_idx, res_val, chunk_ptr, landmark_norm, chunk_pos=None,
                 res_scale=None) -> lowram_cache:
    return lowram_cache(_ptr(coef), _ptr(landmark), _ptr(res_idx), _ptr(res_val),
                        _ptr(chunk_ptr), _ptr(landmark_norm), _ptr(chunk_pos), _ptr(res_scale))


def alloc_cache(cfg: lowram_config, device):
    """Device tensors of one layer's compressed cache (shapes of include/lowram.h)."""
    import torch
    dt = torch.bfloat16 if cfg.dtype == DTYPE_BF16 else torch.float32
    B, T, H, d = cfg.batch, cfg.n_tokens, cfg.n_kv_heads, cfg.head_dim
    nc = T // cfg.chunk
    q4 = cfg.res_format == RES_INT4_G32
    out = {
        "coef": torch.empty(B, T, cfg.rank, dtype=dt, device=device),
        "landmark": torch.empty(B, H, nc, d, dtype=dt, device=device),
        "res_idx": torch.empty(B, H, cfg.n_res, dtype=torch.int32, device=device),
        "res_val": (torch.empty(B, H, cfg.n_res, d // 2, dtype=torch.uint8, device=device) if q4
                    else torch.empty(B, H, cfg.n_res, d, dtype=dt, device=device)),
        "chunk_ptr": torch.empty(B, H, nc + 1, dtype=torch.int32, device=device),
        "landmark_norm": torch.empty(B, H, dtype=torch.float32, device=device),
    }
    if cfg.n_positions > cfg.n_tokens:
        out["chunk_pos"] = torch.empty(B, nc, dtype=torch.int32, device=device)
    if q4:
        out["res_scale"] = torch.empty(B, H, cfg.n_res, d // 32, dtype=torch.float16, device=device)
    return out


def encode(ctx: Context, k_cache, v, params: lowram_layer_params, cache: dict, workspace,
           stream=None) -> None:
    cs = cache_struct(**cache)
    check(lowram_encode(ctx.handle, _ptr(k_cache), _ptr(v), ctypes.byref(params),
                        ctypes.byref(cs), _ptr(workspace), workspace.numel() * workspace.element_size(),
                        _stream(stream)), "lowram_encode")


def decode_step(ctx: Context, cache: dict, params: lowram_layer_params, q, out, workspace,
                sel_out=None, stream=None) -> None:
    cs = cache_struct(**cache)
    check(lowram_decode_step(ctx.handle, ctypes.byref(cs), ctypes.byref(params), _ptr(q),
                             _ptr(out), _ptr(sel_out), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)),
          "lowram_decode_step")


def decode_step_static(ctx: Context, cache: dict, params: lowram_layer_params, q, out,
                       sel_out=None, stream=None) -> None:
    """lowram_decode_step_static: the decode step without a caller workspace (its scratch
    is the library's fixed device array; see include/lowram.h)."""
    cs = cache_struct(**cache)
    check(lowram_decode_step_static(ctx.handle, ctypes.byref(cs), ctypes.byref(params), _ptr(q),
                                    _ptr(out), _ptr(sel_out), _stream(stream)),
          "lowram_decode_step_static")


def select_chunks(ctx: Context, landmark, landmark_norm, q, sel_out, workspace,
                  stream=None) -> None:
    check(lowram_select_chunks(ctx.handle, _ptr(landmark), _ptr(landmark_norm), _ptr(q),
                               _ptr(sel_out), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)),
          "lowram_select_chunks")


def landmark_norms(ctx: Context, landmark, out, stream=None) -> None:
    """lowram_landmark_norms: out [B][H_kv] fp32 = max_c |landmark_c|_2, rounded up."""
    check(lowram_landmark_norms(ctx.handle, _ptr(landmark), _ptr(out), _stream(stream)),
          "lowram_landmark_norms")


def attend_selected(ctx: Context, cache: dict, params: lowram_layer_params, q, sel, out,
                    workspace, stream=None) -> None:
    cs = cache_struct(**cache)
    check(lowram_attend_selected(ctx.handle, ctypes.byref(cs), ctypes.byref(params), _ptr(q),
                                 _ptr(sel), _ptr(out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
          "lowram_attend_selected")


def debug_tc_tile(a, b, d, k: int, mode: int, stream=None) -> None:
    check(lowram_debug_tc_tile(_ptr(a), _ptr(b), _ptr(d), k, mode, _stream(stream)),
          "lowram_debug_tc_tile")


def debug_reconstruct(ctx: Context, cache: dict, params: lowram_layer_params, q, sel, out,
                      k_rot, h_act, v_rec, workspace, stream=None) -> None:
    """Test only: lowram_debug_reconstruct (attend + the rebuilt rows; include/lowram.h)."""
    cs = cache_struct(**cache)
    check(lowram_debug_reconstruct(ctx.handle, ctypes.byref(cs), ctypes.byref(params), _ptr(q),
                                   _ptr(sel), _ptr(out), _ptr(k_rot), _ptr(h_act), _ptr(v_rec),
                                   _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream)),
          "lowram_debug_reconstruct")


def debug_attend_unpublished(ctx: Context, cache: dict, params: lowram_layer_params, q, sel,
                             out, workspace, stream=None) -> None:
    """Test only: lowram_debug_attend_unpublished (a wait that runs out; include/lowram.h)."""
    cs = cache_struct(**cache)
    check(lowram_debug_attend_unpublished(ctx.handle, ctypes.byref(cs), ctypes.byref(params),
                                          _ptr(q), _ptr(sel), _ptr(out), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          _stream(stream)),
          "lowram_debug_attend_unpublished")


def dense_decode(ctx: Context, k_cache, v, q, out, workspace, stream=None) -> None:
    """lowram_dense_decode: exact GQA decode attention over the uncompressed bf16 cache."""
    check(lowram_dense_decode(ctx.handle, _ptr(k_cache), _ptr(v), _ptr(q), _ptr(out),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream)),
          "lowram_dense_decode")


def evict(ctx: Context, k_full, v_full, k_kept, v_kept, chunk_pos, workspace, stream=None) -> None:
    """lowram_evict: keep the chunks with the largest all-head landmark norm (LowRAM-E)."""
    check(lowram_evict(ctx.handle, _ptr(k_full), _ptr(v_full), _ptr(k_kept), _ptr(v_kept),
                       _ptr(chunk_pos), _ptr(workspace),
                       workspace.numel() * workspace.element_size(), _stream(stream)),
          "lowram_evict")


def append(dst_ctx: Context, dst: dict, prefix_ctx: Context, prefix: dict, block_ctx: Context,
           block: dict, stream=None) -> None:
    """lowram_append: the cache of a compressed prefix followed by a compressed block of
    generated tokens (periodic re-compression of the suffix)."""
    cd, cp, cb = cache_struct(**dst), cache_struct(**prefix), cache_struct(**block)
    check(lowram_append(dst_ctx.handle, ctypes.byref(cd), prefix_ctx.handle, ctypes.byref(cp),
                        block_ctx.handle, ctypes.byref(cb), _stream(stream)), "lowram_append")


def fit_basis_workspace_size(cfg: lowram_config, l: int) -> int:
    n = ctypes.c_size_t()
    check(lowram_fit_basis_workspace_size(ctypes.byref(cfg), l, ctypes.byref(n)),
          "lowram_fit_basis_workspace_size")
    return n.value


def fit_basis(ctx: Context, k_layers, omega, n_power: int, basis_out, workspace,
              stream=None) -> None:
    """lowram_fit_basis: the group's xKV basis by a randomised range finder with
    Cholesky-QR. k_layers: list of device tensors [B][T][H][d]; omega [D][l] fp64."""
    arr = (ctypes.c_void_p * len(k_layers))(*[t.data_ptr() for t in k_layers])
    for t in k_layers:
        _ptr(t)   # contiguity check
    check(lowram_fit_basis(ctx.handle, arr, len(k_layers), _ptr(omega), omega.shape[1],
                           n_power, _ptr(basis_out), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream)),
          "lowram_fit_basis")


def suffix_workspace_size(cfg: lowram_config, s_max: int) -> int:
    n = ctypes.c_size_t()
    check(lowram_suffix_workspace_size(ctypes.byref(cfg), s_max, ctypes.byref(n)),
          "lowram_suffix_workspace_size")
    return n.value


def decode_step_suffix(ctx: Context, cache: dict, params: lowram_layer_params, q, k_suffix,
                       v_suffix, n_suffix: int, out, workspace, sel_out=None,
                       stream=None) -> None:
    """lowram_decode_step_suffix: decode over the compressed prefix plus the first n_suffix
    rows of an uncompressed suffix buffer [B][s_max][H][d]."""
    cs = cache_struct(**cache)
    check(lowram_decode_step_suffix(ctx.handle, ctypes.byref(cs), ctypes.byref(params), _ptr(q),
                                    _ptr(k_suffix), _ptr(v_suffix), k_suffix.shape[1], n_suffix,
                                    _ptr(out), _ptr(sel_out), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
          "lowram_decode_step_suffix")
