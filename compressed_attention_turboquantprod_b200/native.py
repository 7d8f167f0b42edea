"""ctypes binding of libtq (include/tq.h): argument marshalling only.

Every function here has the name of the C call it wraps, takes torch tensors
(device memory and streams come from PyTorch) and raises ``TQError`` on a
non-zero status.  No step of the method runs in Python.  Importing this module
fails loudly if ``libtq.so`` is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# TQ_LIBRARY=bounds loads the bounds-checked build (libtq_bounds.so) instead.
LIB_PATH = os.path.join(_HERE, "libtq_bounds.so" if os.environ.get("TQ_LIBRARY") == "bounds"
                        else "libtq.so")

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CAPACITY, TQ_ERR_CUDA, TQ_ERR_NOT_CONVERGED = range(6)
TQ_F32, TQ_F16, TQ_BF16 = 0, 1, 2
BLOCK_TOKENS = 64

_DT = {torch.float32: TQ_F32, torch.float16: TQ_F16, torch.bfloat16: TQ_BF16}


class TQError(RuntimeError):
    def __init__(self, status: int, message: str, call: str):
        super().__init__(f"{call} failed with status {status}: {message}")
        self.status = status
        self.message = message
        self.call = call


class tq_cache_desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32),
                ("b1", ctypes.c_int32), ("m", ctypes.c_int32), ("vbits", ctypes.c_int32),
                ("group", ctypes.c_int32), ("W", ctypes.c_int32), ("capacity", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("rotation", ctypes.c_int32)]


class tq_cache(ctypes.Structure):
    _fields_ = [("desc", tq_cache_desc), ("base", ctypes.c_void_p), ("bytes", ctypes.c_size_t),
                ("n_total", ctypes.c_int64), ("block_bytes", ctypes.c_int64),
                ("region_bytes", ctypes.c_int64), ("ring_k_off", ctypes.c_int64),
                ("ring_v_off", ctypes.c_int64), ("token_bytes", ctypes.c_int32),
                ("o_idx", ctypes.c_int32), ("o_sign", ctypes.c_int32), ("o_rho", ctypes.c_int32),
                ("o_rnorm", ctypes.c_int32), ("o_vcode", ctypes.c_int32),
                ("o_vscale", ctypes.c_int32), ("o_vmin", ctypes.c_int32)]


class tq_layer_groups(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int32), ("bound", ctypes.c_int32 * 8), ("m", ctypes.c_int32 * 8)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libtq.so not built ({LIB_PATH}); run "
                          "`python -m compressed_attention_turboquantprod_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, SZ, U64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t, ctypes.c_uint64)
    C = ctypes.POINTER(tq_cache)
    D = ctypes.POINTER(tq_cache_desc)
    sig = {
        "tq_last_error": (ctypes.c_char_p, []),
        "tq_version": (I, []),
        "tq_debug_fail_next": (I, [ctypes.c_char_p]),
        "tq_debug_bounds_enabled": (I, []),
        "tq_debug_bounds_check": (I, []),
        "tq_codebook_build": (I, [I, I, P, P, P]),
        "tq_projections_workspace_bytes": (SZ, [I]),
        "tq_make_projections": (I, [I, I, I, U64, U64, P, P, P, P, SZ, P]),
        "tq_make_projections_hadamard": (I, [I, I, I, U64, U64, P, P, P, P]),
        "tq_quantize_keys": (I, [P, I, I64, I, I, I, P, P, P, P, P, P, P, P, P]),
        "tq_quantize_values": (I, [P, I, I64, I, I, I, P, P, P, P]),
        "tq_cache_bytes": (SZ, [D]),
        "tq_cache_layout": (I, [D, C]),
        "tq_cache_init": (I, [C, D, P, SZ, P]),
        "tq_cache_compressed_tokens": (I64, [C]),
        "tq_cache_ring_tokens": (I64, [C]),
        "tq_append": (I, [C, P, P, I64, P, P, P, P, P]),
        "tq_decode_auto_splits": (I, [C, I]),
        "tq_decode_workspace_bytes": (SZ, [C, I, I]),
        "tq_decode_attention": (I, [C, P, I, F, P, P, P, P, P, I, P, SZ, P]),
        "tq_decode_attention_noalloc": (I, [C, P, I, F, P, P, P, P, P, I, P]),
        "tq_decode_prep": (I, [C, P, I, F, P, P, P, I, P, SZ, P]),
        "tq_decode_check": (I, [C, I, I, P, SZ, P]),
        "tq_quantize_check": (I, [P]),
        "tq_decode_partial": (I, [C, I, F, P, P, P, I, P, SZ, P]),
        "tq_decode_combine": (I, [C, I, P, I, P, SZ, P]),
        "tq_decode_step": (I, [C, P, P, I64, P, I, F, P, P, P, P, P, P, P, I, P, SZ, P]),
        "tq_prefill_workspace_bytes": (SZ, [C, I, I, I]),
        "tq_prefill_attention": (I, [C, P, I, I, P, P, F, P, P, P, P, I, P, SZ, P]),
        "tq_prefill_check": (I, [C, I, I, I, P, SZ, P]),
        "tq_key_moments_workspace_bytes": (SZ, []),
        "tq_key_moments": (I, [P, I, I64, P, P, SZ, P]),
        "tq_sensitivity_profile": (I, [ctypes.POINTER(ctypes.c_double), I, I, I, I, I,
                                       ctypes.POINTER(tq_layer_groups)]),
        "tq_decode_partials_view": (I, [C, I, I, P, SZ, ctypes.POINTER(P), ctypes.POINTER(P),
                                        ctypes.POINTER(I)]),
        "tq_merge_partials": (I, [P, P, I64, I, I, I, P, P]),
        "tq_layer_groups_parse": (I, [ctypes.c_char_p, ctypes.c_char_p, ctypes.POINTER(tq_layer_groups)]),
        "tq_m_for_layer": (I, [ctypes.POINTER(tq_layer_groups), I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _check(status: int, call: str):
    if status != TQ_OK:
        raise TQError(status, lib.tq_last_error().decode(errors="replace"), call)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def dtype_code(dt: torch.dtype) -> int:
    return _DT[dt]


# ----------------------------------------------------------------------------- setup
def tq_codebook_build(d: int, bits: int, centroids: torch.Tensor, boundaries: torch.Tensor,
                      stream=None):
    _check(lib.tq_codebook_build(d, bits, _ptr(centroids), _ptr(boundaries), _stream(stream)),
           "tq_codebook_build")


def tq_projections_workspace_bytes(d: int) -> int:
    return lib.tq_projections_workspace_bytes(d)


def tq_make_projections(d: int, m: int, layer: int, Pi, S, T, workspace, base_seed: int = 42,
                        stride: int = 7, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.tq_make_projections(d, m, layer, base_seed, stride, _ptr(Pi), _ptr(S), _ptr(T),
                                   _ptr(workspace), ws_bytes, _stream(stream)),
           "tq_make_projections")


def tq_make_projections_hadamard(d: int, m: int, layer: int, Pi, S, T, base_seed: int = 42,
                                 stride: int = 7, stream=None):
    _check(lib.tq_make_projections_hadamard(d, m, layer, base_seed, stride, _ptr(Pi), _ptr(S),
                                            _ptr(T), _stream(stream)),
           "tq_make_projections_hadamard")


# ----------------------------------------------------------------------------- quantise
def tq_quantize_keys(K: torch.Tensor, b1: int, m: int, Pi, T, centroids, boundaries, idx_planes,
                     signs, norm_x, norm_r, stream=None):
    n, d = K.shape
    _check(lib.tq_quantize_keys(_ptr(K), dtype_code(K.dtype), n, d, b1, m, _ptr(Pi), _ptr(T),
                                _ptr(centroids), _ptr(boundaries), _ptr(idx_planes), _ptr(signs),
                                _ptr(norm_x), _ptr(norm_r), _stream(stream)), "tq_quantize_keys")


def tq_quantize_values(V: torch.Tensor, vbits: int, group: int, codes, scale, vmin, stream=None):
    n, d = V.shape
    _check(lib.tq_quantize_values(_ptr(V), dtype_code(V.dtype), n, d, vbits, group, _ptr(codes),
                                  _ptr(scale), _ptr(vmin), _stream(stream)), "tq_quantize_values")


# ----------------------------------------------------------------------------- cache
TQ_ROTATION_DENSE, TQ_ROTATION_HADAMARD = 0, 1


def make_desc(B, Hkv, d, b1, m, vbits, group, W, capacity, dtype,
              rotation=TQ_ROTATION_DENSE) -> tq_cache_desc:
    return tq_cache_desc(B, Hkv, d, b1, m, vbits, group, W, capacity,
                         dtype if isinstance(dtype, int) else dtype_code(dtype), rotation)


def tq_cache_bytes(desc: tq_cache_desc) -> int:
    return lib.tq_cache_bytes(ctypes.byref(desc))


def tq_cache_layout(desc: tq_cache_desc) -> tq_cache:
    c = tq_cache()
    _check(lib.tq_cache_layout(ctypes.byref(desc), ctypes.byref(c)), "tq_cache_layout")
    return c


def tq_cache_init(cache: tq_cache, desc: tq_cache_desc, buf: torch.Tensor, stream=None):
    _check(lib.tq_cache_init(ctypes.byref(cache), ctypes.byref(desc), _ptr(buf),
                             buf.numel() * buf.element_size(), _stream(stream)), "tq_cache_init")


def tq_append(cache: tq_cache, K, V, Pi, T, centroids, boundaries, stream=None):
    n_new = K.shape[2]
    _check(lib.tq_append(ctypes.byref(cache), _ptr(K), _ptr(V), n_new, _ptr(Pi), _ptr(T),
                         _ptr(centroids), _ptr(boundaries), _stream(stream)), "tq_append")


def tq_decode_workspace_bytes(cache: tq_cache, Hq: int, num_splits: int = 0) -> int:
    return lib.tq_decode_workspace_bytes(ctypes.byref(cache), Hq, num_splits)


def tq_decode_auto_splits(cache: tq_cache, Hq: int) -> int:
    return lib.tq_decode_auto_splits(ctypes.byref(cache), Hq)


def _ws(workspace):
    return workspace.numel() * workspace.element_size()


def tq_decode_attention(cache: tq_cache, Q, softmax_scale: float, Pi, S, centroids, out,
                        logits=None, num_splits: int = 0, workspace=None, stream=None):
    Hq = Q.shape[1]
    _check(lib.tq_decode_attention(ctypes.byref(cache), _ptr(Q), Hq, softmax_scale, _ptr(Pi),
                                   _ptr(S), _ptr(centroids), _ptr(out), _ptr(logits), num_splits,
                                   _ptr(workspace), _ws(workspace), _stream(stream)),
           "tq_decode_attention")


def tq_decode_attention_noalloc(cache: tq_cache, Q, softmax_scale: float, Pi, S, centroids, out,
                                logits=None, num_splits: int = 0, stream=None):
    Hq = Q.shape[1]
    _check(lib.tq_decode_attention_noalloc(ctypes.byref(cache), _ptr(Q), Hq, softmax_scale,
                                           _ptr(Pi), _ptr(S), _ptr(centroids), _ptr(out),
                                           _ptr(logits), num_splits, _stream(stream)),
           "tq_decode_attention_noalloc")


def tq_decode_prep(cache: tq_cache, Q, softmax_scale, Pi, S, centroids, num_splits, workspace,
                   stream=None):
    _check(lib.tq_decode_prep(ctypes.byref(cache), _ptr(Q), Q.shape[1], softmax_scale, _ptr(Pi),
                              _ptr(S), _ptr(centroids), num_splits, _ptr(workspace),
                              _ws(workspace), _stream(stream)), "tq_decode_prep")


def tq_prefill_workspace_bytes(cache: tq_cache, Hq: int, n: int, num_splits: int = 0) -> int:
    return lib.tq_prefill_workspace_bytes(ctypes.byref(cache), Hq, n, num_splits)


def tq_prefill_attention(cache: tq_cache, Q, K, V, softmax_scale: float, Pi, S, centroids, out,
                         num_splits: int = 0, workspace=None, stream=None):
    """Q [B, n, Hq, d]; K, V [B, Hkv, n, d]; out [B, n, Hq, d]."""
    n, Hq = Q.shape[1], Q.shape[2]
    _check(lib.tq_prefill_attention(ctypes.byref(cache), _ptr(Q), Hq, n, _ptr(K), _ptr(V),
                                    softmax_scale, _ptr(Pi), _ptr(S), _ptr(centroids), _ptr(out),
                                    num_splits, _ptr(workspace), _ws(workspace), _stream(stream)),
           "tq_prefill_attention")


def tq_prefill_check(cache: tq_cache, Hq, n, num_splits, workspace, stream=None):
    _check(lib.tq_prefill_check(ctypes.byref(cache), Hq, n, num_splits, _ptr(workspace),
                                _ws(workspace), _stream(stream)), "tq_prefill_check")


def tq_quantize_check(stream=None):
    """Raise if the batched tensor-core key quantisation gave up a bounded wait
    since the last check (waits for the stream; clears the flag)."""
    _check(lib.tq_quantize_check(_stream(stream)), "tq_quantize_check")


def tq_decode_check(cache: tq_cache, Hq, num_splits, workspace, stream=None):
    """workspace None: the static scratch of tq_decode_attention_noalloc."""
    _check(lib.tq_decode_check(ctypes.byref(cache), Hq, num_splits, _ptr(workspace),
                               _ws(workspace) if workspace is not None else 0, _stream(stream)),
           "tq_decode_check")


def tq_decode_partial(cache: tq_cache, Hq, softmax_scale, centroids, logits, num_splits,
                      workspace, out=None, stream=None):
    _check(lib.tq_decode_partial(ctypes.byref(cache), Hq, softmax_scale, _ptr(centroids),
                                 _ptr(logits), _ptr(out), num_splits, _ptr(workspace),
                                 _ws(workspace), _stream(stream)), "tq_decode_partial")


def tq_decode_step(cache: tq_cache, K, V, Q, softmax_scale, Pi, S, T, centroids, boundaries, out,
                   logits, num_splits, workspace, stream=None):
    _check(lib.tq_decode_step(ctypes.byref(cache), _ptr(K), _ptr(V), K.shape[2], _ptr(Q), Q.shape[1],
                              softmax_scale, _ptr(Pi), _ptr(S), _ptr(T), _ptr(centroids),
                              _ptr(boundaries), _ptr(out), _ptr(logits), num_splits, _ptr(workspace),
                              _ws(workspace), _stream(stream)), "tq_decode_step")


def tq_decode_combine(cache: tq_cache, Hq, out, num_splits, workspace, stream=None):
    _check(lib.tq_decode_combine(ctypes.byref(cache), Hq, _ptr(out), num_splits, _ptr(workspace),
                                 _ws(workspace), _stream(stream)), "tq_decode_combine")


def tq_decode_partials_view(cache: tq_cache, Hq, num_splits, workspace):
    """(part_ml, part_o) as torch views of the workspace: [B*Hq, S, 2] and [B*Hq, S, d]."""
    ml, o, s = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_int()
    _check(lib.tq_decode_partials_view(ctypes.byref(cache), Hq, num_splits, _ptr(workspace),
                                       _ws(workspace), ctypes.byref(ml), ctypes.byref(o),
                                       ctypes.byref(s)), "tq_decode_partials_view")
    rows, S, d = cache.desc.B * Hq, s.value, cache.desc.d
    base = workspace.data_ptr()
    f = workspace.view(torch.uint8)
    ml_t = f[ml.value - base: ml.value - base + rows * S * 2 * 4].view(torch.float32).view(rows, S, 2)
    o_t = f[o.value - base: o.value - base + rows * S * d * 4].view(torch.float32).view(rows, S, d)
    return ml_t, o_t


def tq_merge_partials(part_ml, part_o, out, stream=None):
    """out [rows, d] from part_ml [rows, slots, 2] and part_o [rows, slots, d] (float32)."""
    rows, slots, d = part_o.shape
    _check(lib.tq_merge_partials(_ptr(part_ml), _ptr(part_o), rows, slots, d, dtype_code(out.dtype),
                                 _ptr(out), _stream(stream)), "tq_merge_partials")


# ----------------------------------------------------------------------------- layer groups
def tq_layer_groups_parse(boundaries: str, sketch_dims: str) -> tq_layer_groups:
    g = tq_layer_groups()
    _check(lib.tq_layer_groups_parse(boundaries.encode(), sketch_dims.encode(), ctypes.byref(g)),
           "tq_layer_groups_parse")
    return g


def tq_key_moments_workspace_bytes() -> int:
    return lib.tq_key_moments_workspace_bytes()


def tq_key_moments(K, out, workspace, stream=None):
    """out (device float64[2]) = sum and sum of squares of every entry of K."""
    _check(lib.tq_key_moments(_ptr(K), dtype_code(K.dtype), K.numel(), _ptr(out), _ptr(workspace),
                              _ws(workspace), _stream(stream)), "tq_key_moments")


def tq_sensitivity_profile(layer_var, num_groups: int, m_avg: int, m_min: int = 32,
                           m_max: int = 1024) -> tq_layer_groups:
    L = len(layer_var)
    arr = (ctypes.c_double * L)(*[float(x) for x in layer_var])
    g = tq_layer_groups()
    _check(lib.tq_sensitivity_profile(arr, L, num_groups, m_avg, m_min, m_max, ctypes.byref(g)),
           "tq_sensitivity_profile")
    return g


def tq_m_for_layer(groups: tq_layer_groups, layer: int) -> int:
    return lib.tq_m_for_layer(ctypes.byref(groups), layer)


def tq_debug_fail_next(name: Optional[str]):
    lib.tq_debug_fail_next(name.encode() if name else None)


def tq_debug_bounds_enabled() -> int:
    return lib.tq_debug_bounds_enabled()


def tq_debug_bounds_check():
    _check(lib.tq_debug_bounds_check(), "tq_debug_bounds_check")
