"""ctypes binding of libsemkv (include/semkv.h): argument marshalling only.

Every function here has the name of the C entry point it calls and passes device pointers taken
from torch tensors plus the current CUDA stream; all computation happens in the library's
kernels.  The library must have been built (``python -m mixed_precision_kv_semkv_b200.build``);
there is no fallback: a missing library raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("SEMKV_LIB") or os.path.join(_PKG, "libsemkv.so")  # SEMKV_LIB: another build

SEMKV_OK = 0
SEMKV_ERR_INVALID_ARG = 1
SEMKV_ERR_UNSUPPORTED = 2
SEMKV_ERR_CAPACITY = 3
SEMKV_ERR_CUDA = 4

STATUS_NAN_SCORE = 1
STATUS_NONFINITE_KV = 2
STATUS_APPEND_OVERFLOW = 4
STATUS_LENGTH_MISMATCH = 8
STATUS_TIMEOUT = 16

SHAPE_FIELDS = ("B", "H", "Hq", "D", "G", "L_hi", "L_lo", "cap_hi", "cap_lo", "T_cap")
BUF_NAMES = ("k_hi", "v_hi", "kz_hi", "vz_hi", "k_lo", "v_lo", "kz_lo", "vz_lo",
             "bitmap", "rank", "n_hi", "n_lo", "tau", "status", "slot_token", "score_keys", "kc")
EXPORTED = ("semkv_cache_bytes", "semkv_workspace_bytes", "semkv_assign_precision", "semkv_quantize_pack",
            "semkv_append_token", "semkv_append_token_running", "semkv_append_decode", "semkv_decode_attention",
            "semkv_decode_attention_noalloc", "semkv_dequantize", "semkv_status_string", "semkv_radix_digits",
            "semkv_p_for_ratio", "semkv_p_for_ratio_kv", "semkv_capacities", "semkv_selftest_wait_timeout")
NOALLOC_SCRATCH_BYTES = 4 << 20  # SEMKV_NOALLOC_SCRATCH_BYTES


class CacheStruct(ctypes.Structure):
    """Mirror of semkv_cache_t (window, clip, L_hi_v, L_lo_v, k_per_channel: the quantizer variants;
    0 = off)."""
    _fields_ = [(n, ctypes.c_int32) for n in SHAPE_FIELDS] + \
        [("window", ctypes.c_int32), ("clip", ctypes.c_float), ("L_hi_v", ctypes.c_int32), ("L_lo_v", ctypes.c_int32),
         ("k_per_channel", ctypes.c_int32)] + \
        [(n, ctypes.c_void_p) for n in BUF_NAMES]


class SemkvError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {code} ({status_string(code)})")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libsemkv.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m mixed_precision_kv_semkv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        cp = ctypes.POINTER(CacheStruct)
        vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
        L.semkv_cache_bytes.argtypes = [cp, ctypes.POINTER(sz)]
        L.semkv_workspace_bytes.argtypes = [cp, ctypes.POINTER(sz)]
        L.semkv_assign_precision.argtypes = [cp, vp, i32, f32, vp]
        L.semkv_quantize_pack.argtypes = [cp, vp, vp, i32, vp]
        L.semkv_append_token.argtypes = [cp, vp, vp, vp, vp]
        L.semkv_append_token_running.argtypes = [cp, vp, vp, vp, f32, vp]
        L.semkv_append_decode.argtypes = [cp, vp, vp, vp, vp, f32, vp, vp, sz, vp]
        L.semkv_decode_attention.argtypes = [cp, vp, f32, vp, vp, sz, vp]
        L.semkv_decode_attention_noalloc.argtypes = [cp, vp, f32, vp, vp]
        L.semkv_dequantize.argtypes = [cp, vp, vp, i32, vp]
        L.semkv_status_string.argtypes = [ctypes.c_int]
        L.semkv_status_string.restype = ctypes.c_char_p
        L.semkv_radix_digits.argtypes = [i32]
        L.semkv_radix_digits.restype = i32
        L.semkv_p_for_ratio.argtypes = [i32, i32, i32, i32, ctypes.c_double, ctypes.POINTER(ctypes.c_double)]
        L.semkv_p_for_ratio_kv.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.c_double,
                                           ctypes.POINTER(ctypes.c_double)]
        i32p = ctypes.POINTER(i32)
        L.semkv_capacities.argtypes = [i32, f32, i32, i32, i32p, i32p, i32p, i32p]
        L.semkv_selftest_wait_timeout.argtypes = [vp, i32, i32, vp]
        for n in EXPORTED:
            if n not in ("semkv_status_string", "semkv_radix_digits"):
                getattr(L, n).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().semkv_status_string(int(code)).decode()


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else int(t.data_ptr()))


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        import torch

        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, rc: int) -> int:
    if rc != SEMKV_OK:
        raise SemkvError(fn, rc)
    return rc


def _struct(cache) -> CacheStruct:
    return cache.struct if hasattr(cache, "struct") else cache


def semkv_radix_digits(L: int) -> int:
    return int(lib().semkv_radix_digits(int(L)))


def semkv_p_for_ratio(D: int, G: int, L_hi: int, L_lo: int, ratio: float) -> float:
    """Largest fraction p on the L_hi grid whose storage reduction vs fp16 is still >= ratio."""
    p = ctypes.c_double()
    _check("semkv_p_for_ratio", lib().semkv_p_for_ratio(int(D), int(G), int(L_hi), int(L_lo), float(ratio),
                                                       ctypes.byref(p)))
    return p.value


def semkv_p_for_ratio_kv(D: int, G: int, L_hi: int, L_lo: int, L_hi_v: int, L_lo_v: int, ratio: float) -> float:
    """semkv_p_for_ratio with V level counts of their own."""
    p = ctypes.c_double()
    _check("semkv_p_for_ratio_kv", lib().semkv_p_for_ratio_kv(int(D), int(G), int(L_hi), int(L_lo), int(L_hi_v),
                                                             int(L_lo_v), float(ratio), ctypes.byref(p)))
    return p.value


def semkv_capacities(T: int, p: float, window: int = 0, extra: int = 0) -> tuple[int, int, int, int]:
    """(n_sel, cap_hi, cap_lo, T_cap) of a cache for a prefill of T tokens at fraction p, with the
    last `window` tokens also on the finer grid and room for `extra` appended tokens per unit."""
    out = [ctypes.c_int32() for _ in range(4)]
    _check("semkv_capacities", lib().semkv_capacities(int(T), float(p), int(window), int(extra),
                                                      *(ctypes.byref(o) for o in out)))
    return tuple(int(o.value) for o in out)


def semkv_cache_bytes(cache) -> list[int]:
    sizes = (ctypes.c_size_t * len(BUF_NAMES))()
    _check("semkv_cache_bytes", lib().semkv_cache_bytes(ctypes.byref(_struct(cache)), sizes))
    return list(sizes)


def semkv_workspace_bytes(cache) -> int:
    n = ctypes.c_size_t(0)
    _check("semkv_workspace_bytes", lib().semkv_workspace_bytes(ctypes.byref(_struct(cache)), ctypes.byref(n)))
    return int(n.value)


def semkv_assign_precision(cache, scores, T: int, p: float, stream=None) -> int:
    return _check("semkv_assign_precision",
                  lib().semkv_assign_precision(ctypes.byref(_struct(cache)), _ptr(scores), int(T), float(p),
                                               _stream(stream)))


def semkv_quantize_pack(cache, K, V, T: int, stream=None) -> int:
    return _check("semkv_quantize_pack",
                  lib().semkv_quantize_pack(ctypes.byref(_struct(cache)), _ptr(K), _ptr(V), int(T), _stream(stream)))


def semkv_append_token(cache, k, v, score, stream=None) -> int:
    return _check("semkv_append_token",
                  lib().semkv_append_token(ctypes.byref(_struct(cache)), _ptr(k), _ptr(v), _ptr(score),
                                           _stream(stream)))


def semkv_append_token_running(cache, k, v, score, p: float, stream=None) -> int:
    return _check("semkv_append_token_running",
                  lib().semkv_append_token_running(ctypes.byref(_struct(cache)), _ptr(k), _ptr(v), _ptr(score),
                                                   float(p), _stream(stream)))


def semkv_append_decode(cache, k, v, score, q, softmax_scale: float, out, workspace,
                        workspace_bytes: int | None = None, stream=None) -> int:
    """append_token then decode_attention in one pass over the cache."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _check("semkv_append_decode",
                  lib().semkv_append_decode(ctypes.byref(_struct(cache)), _ptr(k), _ptr(v), _ptr(score), _ptr(q),
                                            float(softmax_scale), _ptr(out), _ptr(workspace), int(workspace_bytes),
                                            _stream(stream)))


def semkv_decode_attention(cache, q, softmax_scale: float, out, workspace, workspace_bytes: int | None = None,
                           stream=None) -> int:
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else int(workspace_bytes)
    return _check("semkv_decode_attention",
                  lib().semkv_decode_attention(ctypes.byref(_struct(cache)), _ptr(q), float(softmax_scale), _ptr(out),
                                               _ptr(workspace), nbytes, _stream(stream)))


def semkv_decode_attention_noalloc(cache, q, softmax_scale: float, out, stream=None) -> int:
    """Decode attention using the library's fixed device scratch instead of a workspace (for
    callers that cannot allocate device memory when they decode)."""
    return _check("semkv_decode_attention_noalloc",
                  lib().semkv_decode_attention_noalloc(ctypes.byref(_struct(cache)), _ptr(q), float(softmax_scale),
                                                       _ptr(out), _stream(stream)))


def semkv_dequantize(cache, K, V, T: int, stream=None) -> int:
    return _check("semkv_dequantize",
                  lib().semkv_dequantize(ctypes.byref(_struct(cache)), _ptr(K), _ptr(V), int(T), _stream(stream)))


def semkv_selftest_wait_timeout(status, tests: int = 16, use_tmem: bool = True, stream=None) -> None:
    """Launch the bounded-wait self-test: a kernel whose wait nothing completes gives up after
    `tests` tests and ORs SEMKV_STATUS_TIMEOUT into `status` (a device int32 tensor of one element)."""
    _check("semkv_selftest_wait_timeout",
           lib().semkv_selftest_wait_timeout(_ptr(status), int(tests), 1 if use_tmem else 0, _stream(stream)))
