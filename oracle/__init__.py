"""CPU oracle for the SemKV hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and its
``--impl reference`` arm) may import this package.  The product library never loads it, and it
imports nothing from the product package.

The arithmetic lives in ``semkv_oracle.c`` (plain C11, built with ``-O2 -ffp-contract=off`` so
that every fp32 operation is one IEEE round-to-nearest operation); this module only builds it
with gcc and marshals numpy arrays through ctypes.  What each function computes, and the passage
of the SemKV page it follows, is documented in the C file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "semkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

TILE = 128  # slots per tile of a segment (layout constant of the oracle's own layout)

_u32p = np.ctypeslib.ndpointer(dtype=np.uint32, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_c = ctypes


def build(force: bool = False) -> str:
    """Compile semkv_oracle.c into liboracle.so next to it (gcc, no fast-math, no contraction)."""
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            tmp = _LIB + f".tmp{os.getpid()}"
            cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                   "-o", tmp, _SRC, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_radix_digits.argtypes = [_c.c_int]
        L.oracle_radix_digits.restype = _c.c_int
        L.oracle_words_per_row.argtypes = [_c.c_int, _c.c_int]
        L.oracle_words_per_row.restype = _c.c_int
        L.oracle_words_per_tile_column.argtypes = [_c.c_int]
        L.oracle_words_per_tile_column.restype = _c.c_int
        L.oracle_half_to_float_array.argtypes = [_u16p, _f32p, _c.c_int64]
        L.oracle_float_to_half_up_array.argtypes = [_f32p, _u16p, _c.c_int64]
        L.oracle_scale_half.argtypes = [_c.c_float]
        L.oracle_scale_half.restype = _c.c_uint16
        L.oracle_n_hi.argtypes = [_c.c_float, _c.c_int32]
        L.oracle_n_hi.restype = _c.c_int32
        L.oracle_select.argtypes = [_f32p, _c.c_int32, _c.c_float, _c.c_int32, _u32p, _u32p,
                                    _c.POINTER(_c.c_int32), _c.POINTER(_c.c_float)]
        L.oracle_select.restype = _c.c_int
        L.oracle_quantize_group.argtypes = [_u16p, _c.c_int, _c.c_int, _u8p,
                                            _c.POINTER(_c.c_uint16), _c.POINTER(_c.c_uint16)]
        L.oracle_quantize_group.restype = _c.c_int
        L.oracle_quantize_group_clip.argtypes = [_u16p, _c.c_int, _c.c_int, _c.c_float, _u8p,
                                                 _c.POINTER(_c.c_uint16), _c.POINTER(_c.c_uint16)]
        L.oracle_quantize_group_clip.restype = _c.c_int
        L.oracle_float_to_half_rn.argtypes = [_c.c_float]
        L.oracle_float_to_half_rn.restype = _c.c_uint16
        L.oracle_pack_word.argtypes = [_u8p, _c.c_int, _c.c_int]
        L.oracle_pack_word.restype = _c.c_uint32
        L.oracle_unpack_word.argtypes = [_c.c_uint32, _c.c_int, _c.c_int, _u8p]
        _u32p_or_null = _c.c_void_p
        L.oracle_quantize_pack_unit.argtypes = [_u16p, _u16p, _c.c_int32, _c.c_int, _c.c_int, _c.c_int,
                                                _c.c_int, _c.c_int, _c.c_int, _c.c_float, _u32p, _c.c_int,
                                                _c.c_int] + [_u32p] * 8 + [_u32p_or_null]
        L.oracle_k_channel_grid.argtypes = [_u16p, _c.c_int32, _c.c_int, _c.c_int, _c.c_int, _c.c_float, _u32p]
        L.oracle_k_channel_grid.restype = _c.c_int
        L.oracle_code_on_grid.argtypes = [_c.c_uint16, _c.c_uint16, _c.c_uint16, _c.c_int]
        L.oracle_code_on_grid.restype = _c.c_int
        L.oracle_quantize_pack_unit.restype = _c.c_int
        L.oracle_dequantize_unit.argtypes = [_c.c_int32, _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_int,
                                             _u32p] + [_u32p] * 8 + [_f32p, _f32p, _c.c_void_p]
        L.oracle_append_unit.argtypes = [_u16p, _u16p, _c.c_float, _c.c_float, _c.c_int, _c.c_int, _c.c_int,
                                         _c.c_int, _c.c_int, _c.c_int, _c.c_float, _c.c_int32, _u32p, _u32p, _c.POINTER(_c.c_int32),
                                         _c.POINTER(_c.c_int32), _c.c_int, _c.c_int] + [_u32p] * 8 + [_c.c_void_p]
        L.oracle_append_unit.restype = _c.c_int
        L.oracle_attention_fp64.argtypes = [_u16p, _c.c_int, _f32p, _f32p, _c.c_int32, _c.c_int, _c.c_float,
                                            _f64p]
        L.oracle_attention_f32.argtypes = [_u16p, _c.c_int, _f32p, _f32p, _c.c_int32, _c.c_int, _c.c_float,
                                           _f32p]
        _lib = L
    return _lib


# status bits of the oracle (same meanings as the library's device status word)
NAN_SCORE = 1
NONFINITE_KV = 2
OVERFLOW = 4
BAD_ARG = 256


def radix_digits(L: int) -> int:
    return lib().oracle_radix_digits(L)


def words_per_row(L: int, D: int) -> int:
    return lib().oracle_words_per_row(L, D)


def words_per_tile_column(L: int) -> int:
    return lib().oracle_words_per_tile_column(L)


def half_to_float(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().oracle_half_to_float_array(h.ravel(), out.ravel(), h.size)
    return out


def float_to_half_up(f) -> np.ndarray:
    f = np.ascontiguousarray(f, dtype=np.float32)
    out = np.empty(f.shape, np.uint16)
    lib().oracle_float_to_half_up_array(f.ravel(), out.ravel(), f.size)
    return out


def half_rn(f: float) -> int:
    """binary16 bits nearest to the fp32 value f (ties to even)."""
    return int(lib().oracle_float_to_half_rn(float(f)))


def scale_half(sf: float) -> int:
    return int(lib().oracle_scale_half(float(sf)))


def n_hi(p: float, T: int) -> int:
    return int(lib().oracle_n_hi(float(p), int(T)))


def select(score, p: float, window: int = 0):
    """Precision assignment of one unit (window: the last `window` tokens also go to the finer
    grid). Returns (bitmap, rank, n_hi, tau, status)."""
    score = np.ascontiguousarray(score, dtype=np.float32)
    T = score.shape[0]
    nw = max((T + 31) // 32, 1)
    bitmap = np.zeros(nw, np.uint32)
    rank = np.zeros(nw, np.uint32)
    nh = _c.c_int32(0)
    tau = _c.c_float(0)
    st = lib().oracle_select(score, T, float(p), int(window), bitmap, rank, _c.byref(nh), _c.byref(tau))
    nwt = (T + 31) // 32
    return bitmap[:nwt], rank[:nwt], nh.value, np.float32(tau.value), st


def quantize_group(x16, L: int, clip: float = 1.0):
    """Quantize one group of fp16 bit patterns (clip in (0, 1]: the clipped-range variant).
    Returns (codes uint8, scale16, zero16, status)."""
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    codes = np.zeros(x16.shape[0], np.uint8)
    s = _c.c_uint16(0)
    z = _c.c_uint16(0)
    st = lib().oracle_quantize_group_clip(x16, x16.shape[0], L, float(clip), codes, _c.byref(s), _c.byref(z))
    return codes, s.value, z.value, st


def pack_word(codes, L: int) -> int:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    return int(lib().oracle_pack_word(codes, codes.shape[0], L))


def unpack_word(w: int, k: int, L: int) -> np.ndarray:
    out = np.zeros(k, np.uint8)
    lib().oracle_unpack_word(int(w) & 0xFFFFFFFF, k, L, out)
    return out


def segment_shapes(D: int, G: int, L: int, tiles: int, Lv: int | None = None):
    """Shapes of one segment's four buffers in the oracle's layout (Lv: the V level count, if not L)."""
    WK = words_per_row(L, D)
    WV = words_per_tile_column(Lv or L)
    ng = D // G
    return {"k": (tiles, WK, TILE), "v": (tiles, WV, D), "kz": (tiles, ng, TILE), "vz": (tiles, ng, TILE)}


def _alloc_unit(D, G, L_hi, L_lo, tiles_hi, tiles_lo, L_hi_v=None, L_lo_v=None):
    hi = {n: np.zeros(s, np.uint32) for n, s in segment_shapes(D, G, L_hi, tiles_hi, L_hi_v).items()}
    lo = {n: np.zeros(s, np.uint32) for n, s in segment_shapes(D, G, L_lo, tiles_lo, L_lo_v).items()}
    return hi, lo


def _seg_args(hi, lo):
    return [hi["k"].ravel(), hi["v"].ravel(), hi["kz"].ravel(), hi["vz"].ravel(),
            lo["k"].ravel(), lo["v"].ravel(), lo["kz"].ravel(), lo["vz"].ravel()]


def _ptr_or_null(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.uint32).ctypes.data


def k_channel_grid(K16, L_hi: int, L_lo: int, clip: float = 1.0):
    """Per-channel K grids of one unit: uint32 [2][D] (hi, lo; fp16 scale | fp16 zero << 16) and status."""
    K16 = np.ascontiguousarray(K16, dtype=np.uint16)
    T, D = K16.shape
    kc = np.zeros((2, D), np.uint32)
    st = lib().oracle_k_channel_grid(K16.ravel() if T else np.zeros(1, np.uint16), T, D, L_hi, L_lo, float(clip),
                                     kc.ravel())
    return kc, st


def code_on_grid(x16: int, s16: int, z16: int, L: int) -> int:
    return int(lib().oracle_code_on_grid(int(x16), int(s16), int(z16), int(L)))


def quantize_pack_unit(K16, V16, bitmap, G: int, L_hi: int, L_lo: int, tiles_hi: int, tiles_lo: int,
                       clip: float = 1.0, L_hi_v: int | None = None, L_lo_v: int | None = None, kc=None):
    """Quantize and place one unit. K16, V16: [T][D] uint16.  L_hi_v, L_lo_v: V level counts of the
    two segments (default: the K ones).  kc: per-channel K grids (k_channel_grid), or None for
    per-token K groups. Returns (hi, lo, status)."""
    K16 = np.ascontiguousarray(K16, dtype=np.uint16)
    V16 = np.ascontiguousarray(V16, dtype=np.uint16)
    T, D = K16.shape
    L_hi_v, L_lo_v = L_hi_v or L_hi, L_lo_v or L_lo
    hi, lo = _alloc_unit(D, G, L_hi, L_lo, tiles_hi, tiles_lo, L_hi_v, L_lo_v)
    bm = np.zeros(max((T + 31) // 32, 1), np.uint32)
    n = min(len(bitmap), len(bm))
    bm[:n] = bitmap[:n]
    kc = None if kc is None else np.ascontiguousarray(kc, dtype=np.uint32)
    st = lib().oracle_quantize_pack_unit(K16.ravel(), V16.ravel(), T, D, G, L_hi, L_lo, L_hi_v, L_lo_v, float(clip),
                                         bm, tiles_hi, tiles_lo,
                                         *_seg_args(hi, lo), _ptr_or_null(kc))
    return hi, lo, st


def dequantize_unit(T: int, D: int, G: int, L_hi: int, L_lo: int, bitmap, hi, lo, L_hi_v: int | None = None,
                    L_lo_v: int | None = None, kc=None):
    """Dequantize one unit back to original token order. Returns (Khat, Vhat) fp32 [T][D]."""
    Kh = np.zeros((max(T, 1), D), np.float32)
    Vh = np.zeros((max(T, 1), D), np.float32)
    bm = np.zeros(max((T + 31) // 32, 1), np.uint32)
    n = min(len(bitmap), len(bm))
    bm[:n] = bitmap[:n]
    kc = None if kc is None else np.ascontiguousarray(kc, dtype=np.uint32)
    lib().oracle_dequantize_unit(T, D, G, L_hi, L_lo, L_hi_v or L_hi, L_lo_v or L_lo, bm, *_seg_args(hi, lo),
                                 Kh.ravel(), Vh.ravel(), _ptr_or_null(kc))
    return Kh[:T], Vh[:T]


class UnitState:
    """Mutable state of one unit for the append path (bitmap, rank, counts, segments)."""

    def __init__(self, T_cap, bitmap, rank, n_hi, n_lo, tau, hi, lo, kc=None):
        nw = (T_cap + 31) // 32
        self.T_cap = T_cap
        self.bitmap = np.zeros(nw, np.uint32)
        self.bitmap[: len(bitmap)] = bitmap
        self.rank = np.zeros(nw, np.uint32)
        self.rank[: len(rank)] = rank
        self.n_hi = int(n_hi)
        self.n_lo = int(n_lo)
        self.tau = np.float32(tau)
        self.hi = hi
        self.lo = lo
        self.kc = None if kc is None else np.ascontiguousarray(kc, dtype=np.uint32)  # per-channel K grids


def append_unit(state: UnitState, k16, v16, score: float, G: int, L_hi: int, L_lo: int, clip: float = 1.0,
                L_hi_v: int | None = None, L_lo_v: int | None = None) -> int:
    """Append one token to a unit in place (clip, V level counts: as in quantize_pack_unit).
    Returns status bits."""
    k16 = np.ascontiguousarray(k16, dtype=np.uint16)
    v16 = np.ascontiguousarray(v16, dtype=np.uint16)
    D = k16.shape[0]
    nh = _c.c_int32(state.n_hi)
    nl = _c.c_int32(state.n_lo)
    st = lib().oracle_append_unit(k16, v16, float(score), float(state.tau), D, G, L_hi, L_lo, L_hi_v or L_hi,
                                  L_lo_v or L_lo, float(clip), state.T_cap,
                                  state.bitmap, state.rank, _c.byref(nh), _c.byref(nl),
                                  state.hi["k"].shape[0], state.lo["k"].shape[0], *_seg_args(state.hi, state.lo),
                                  _ptr_or_null(state.kc))
    state.n_hi = nh.value
    state.n_lo = nl.value
    return st


def attention_fp64(q16, Khat, Vhat, sm_scale: float) -> np.ndarray:
    """fp64 GQA decode attention of one unit. q16: [g][D] uint16; Khat, Vhat: [T][D] fp32."""
    q16 = np.ascontiguousarray(q16, dtype=np.uint16)
    g, D = q16.shape
    Kh = np.ascontiguousarray(Khat, dtype=np.float32)
    Vh = np.ascontiguousarray(Vhat, dtype=np.float32)
    T = Kh.shape[0]
    if T == 0:
        Kh = np.zeros((1, D), np.float32)
        Vh = np.zeros((1, D), np.float32)
    out = np.zeros((g, D), np.float64)
    lib().oracle_attention_fp64(q16.ravel(), g, Kh.ravel(), Vh.ravel(), T, D, float(sm_scale), out.ravel())
    return out


def attention_f32(q16, Khat, Vhat, sm_scale: float) -> np.ndarray:
    """The same attention with binary32 arithmetic and accumulation (the timed CPU baseline; parity
    is taken against attention_fp64). q16: [g][D] uint16; Khat, Vhat: [T][D] fp32."""
    q16 = np.ascontiguousarray(q16, dtype=np.uint16)
    g, D = q16.shape
    Kh = np.ascontiguousarray(Khat, dtype=np.float32)
    Vh = np.ascontiguousarray(Vhat, dtype=np.float32)
    T = Kh.shape[0]
    if T == 0:
        Kh = np.zeros((1, D), np.float32)
        Vh = np.zeros((1, D), np.float32)
    out = np.zeros((g, D), np.float32)
    lib().oracle_attention_f32(q16.ravel(), g, Kh.ravel(), Vh.ravel(), T, D, float(sm_scale), out.ravel())
    return out


def running_is_hi(scores_prev, score_new: float, p: float) -> bool:
    """Exact running top-p for a generated token (reading of the running threshold): select again
    over all T + 1 scores, the new token last, and read the new token's bit.  Earlier tokens keep
    their grid; only the new token's assignment is taken from this selection."""
    allsc = np.concatenate([np.asarray(scores_prev, np.float32), np.float32([score_new])])
    T = allsc.shape[0] - 1
    bm, _, _, _, _ = select(allsc, p)
    return bool((int(bm[T // 32]) >> (T % 32)) & 1)


def append_unit_running(state: UnitState, k16, v16, score: float, p: float, scores_prev, G: int, L_hi: int,
                        L_lo: int, clip: float = 1.0, L_hi_v: int | None = None, L_lo_v: int | None = None) -> int:
    """append_unit with the running top-p rule: the grid comes from running_is_hi (the fixed tau
    of the state is left as it was)."""
    tau = state.tau
    state.tau = np.float32(-np.inf) if running_is_hi(scores_prev, score, p) else np.float32(np.inf)
    try:
        return append_unit(state, k16, v16, score, G, L_hi, L_lo, clip, L_hi_v, L_lo_v)
    finally:
        state.tau = tau


def p_for_ratio(D: int, G: int, L_hi: int, L_lo: int, ratio: float, iters: int = 200, L_hi_v: int | None = None,
                L_lo_v: int | None = None):
    """Largest fraction p in [0, 1] of tokens on the L_hi grid whose storage reduction against
    fp16 (16 bits / storage_bits_per_value) is still at least `ratio`; None if even p = 0 misses
    it.  SemKV page, Abstract: the recipe is to measure the quality cliff and then interpolate
    above it -- the finer grid's share is what a storage budget leaves room for.  Plain bisection
    on the buffer-derived storage above (no closed-form inversion)."""
    if not ratio > 0.0:
        return None
    ok = lambda p: 16.0 / storage_bits_per_value(D, G, L_hi, L_lo, p, L_hi_v, L_lo_v) >= ratio  # noqa: E731
    if ok(1.0):
        return 1.0
    if not ok(0.0):
        return None
    lo, hi = 0.0, 1.0  # ok(lo), not ok(hi)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if ok(mid):
            lo = mid
        else:
            hi = mid
        if hi - lo < 1e-15:
            break
    return lo


def storage_bits_per_value(D: int, G: int, L_hi: int, L_lo: int, p_real: float, L_hi_v: int | None = None,
                           L_lo_v: int | None = None) -> float:
    """Physical bits per cached value (K and V averaged), from the oracle's own buffer sizes per
    full tile.

    Counts the packed code words of K and of V (each with its own level count), the fp16 scale +
    fp16 zero per group and the one-bit precision bitmap (shared by K and V, so half a bit per
    token per channel pair / D).
    """
    def seg_bits(L, Lv):
        sh = segment_shapes(D, G, L, 1, Lv)
        words_k = int(np.prod(sh["k"]))     # one tile of K rows: 128 tokens x D channels
        words_v = int(np.prod(sh["v"]))     # one tile of V columns: the same 128 x D values
        words_sz = int(np.prod(sh["kz"]))   # per tensor
        return ((words_k + words_v) / 2 + words_sz) * 32 / (TILE * D)
    return p_real * seg_bits(L_hi, L_hi_v or L_hi) + (1 - p_real) * seg_bits(L_lo, L_lo_v or L_lo) + 1.0 / (2 * D)
