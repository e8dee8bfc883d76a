"""Host-side checks of the C ABI that need no GPU: the library loads, exports every entry point
declared in include/*.h, reports buffer sizes that match the oracle's independent layout, and
rejects bad arguments before any CUDA call."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"SEMKV_API\s+[\w\s\*]+?\b(semkv_\w+)\s*\(", src))
    return names


def test_library_exports_every_declared_entry_point(semkv):
    declared = _declared_symbols()
    assert {"semkv_assign_precision", "semkv_quantize_pack", "semkv_append_token", "semkv_decode_attention",
            "semkv_dequantize"} <= declared
    lib = ctypes.CDLL(semkv._lib.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


def _shape(**kw):
    from mixed_precision_kv_semkv_b200 import _lib

    base = dict(B=2, H=8, Hq=32, D=128, G=64, L_hi=8, L_lo=5, cap_hi=256, cap_lo=768, T_cap=1024)
    base.update(kw)
    return _lib.CacheStruct(**base)


def test_radix_digits_agree_with_oracle(semkv, orc):
    for L in range(2, 257):
        assert semkv.semkv_radix_digits(L) == orc.radix_digits(L)
    assert semkv.semkv_radix_digits(1) == 0 and semkv.semkv_radix_digits(257) == 0


@pytest.mark.parametrize("L_hi,L_lo,G", [(8, 5, 64), (6, 5, 128), (16, 8, 32), (3, 2, 8), (256, 17, 16)])
def test_cache_bytes_match_oracle_layout(semkv, orc, L_hi, L_lo, G):
    s = _shape(L_hi=L_hi, L_lo=L_lo, G=G)
    sizes = dict(zip(semkv._lib.BUF_NAMES, semkv.semkv_cache_bytes(s)))
    units = 2 * 8
    for seg, L, cap in (("hi", L_hi, 256), ("lo", L_lo, 768)):
        sh = orc.segment_shapes(128, G, L, cap // 128)
        for name in ("k", "v", "kz", "vz"):
            n = 1
            for x in sh[name]:
                n *= x
            assert sizes[f"{name}_{seg}"] == units * n * 4
    assert sizes["bitmap"] == sizes["rank"] == units * 1024 // 32 * 4
    assert sizes["n_hi"] == sizes["n_lo"] == sizes["tau"] == units * 4
    assert sizes["status"] == 4
    assert sizes["slot_token"] == units * (256 + 768) * 4
    assert sizes["score_keys"] == units * 1024 * 4
    assert sizes["kc"] == units * 2 * 128 * 4  # per-channel K grids: hi and lo per channel


@pytest.mark.parametrize("bad,code", [
    (dict(Hq=30), 1), (dict(G=48), 1), (dict(cap_hi=100), 1), (dict(T_cap=1000), 1), (dict(B=0), 1),
    (dict(D=64, G=64), 2), (dict(L_hi=257), 2), (dict(L_lo=1), 2), (dict(G=4), 2), (dict(Hq=8 * 16), 2),
    (dict(window=-1), 1), (dict(clip=1.5), 1), (dict(clip=-0.25), 1), (dict(clip=float("nan")), 1),
    (dict(L_hi_v=1), 2), (dict(L_lo_v=257), 2), (dict(L_hi_v=-3), 2), (dict(k_per_channel=2), 1),
    (dict(k_per_channel=-1), 1),
])
def test_bad_shapes_are_rejected(semkv, bad, code):
    with pytest.raises(semkv.SemkvError) as e:
        semkv.semkv_cache_bytes(_shape(**bad))
    assert e.value.code == code


def _fake_ptrs(s):
    from mixed_precision_kv_semkv_b200 import _lib

    for i, n in enumerate(_lib.BUF_NAMES):
        setattr(s, n, 0x1000 * (i + 1))  # never dereferenced: every call below fails validation first
    return s


def test_calls_fail_before_any_launch(semkv):
    from mixed_precision_kv_semkv_b200 import _lib

    L = _lib.lib()
    s = _shape()
    ref = ctypes.byref(s)
    nul = ctypes.c_void_p(0)
    one = ctypes.c_void_p(0x1000)
    # null cache pointers
    assert L.semkv_assign_precision(ref, one, 100, 0.25, nul) == 1
    _fake_ptrs(s)
    assert L.semkv_assign_precision(ref, one, 100, 1.5, nul) == 1       # p outside [0, 1]
    assert L.semkv_assign_precision(ref, one, 100, float("nan"), nul) == 1
    assert L.semkv_assign_precision(ref, one, 2000, 0.25, nul) == 1     # T > T_cap
    assert L.semkv_assign_precision(ref, nul, 100, 0.25, nul) == 1      # null scores
    assert L.semkv_assign_precision(ref, one, 1024, 0.5, nul) == 3      # n_hi = 512 > cap_hi = 256
    s.window = 1
    assert L.semkv_assign_precision(ref, one, 1024, 0.25, nul) == 3     # 256 selected + 1 window > 256
    s.window = 0
    assert L.semkv_quantize_pack(ref, nul, one, 10, nul) == 1
    assert L.semkv_append_token(ref, one, one, nul, nul) == 1
    assert L.semkv_decode_attention(ref, one, ctypes.c_float(float("inf")), one, one, 1 << 30, nul) == 1
    assert L.semkv_decode_attention(ref, one, ctypes.c_float(0.1), one, one, 0, nul) == 1  # workspace too small
    assert L.semkv_dequantize(ref, one, nul, 10, nul) == 1
    # append_decode checks the decode's arguments before it appends (on every path)
    sc = ctypes.c_float(0.1)
    assert L.semkv_append_decode(ref, one, one, one, nul, sc, one, one, 1 << 30, nul) == 1   # null q
    assert L.semkv_append_decode(ref, one, one, one, one, sc, one, one, 0, nul) == 1         # workspace too small
    assert L.semkv_append_decode(ref, one, one, one, ctypes.c_void_p(0x1008), sc, one, one, 1 << 30, nul) == 1  # q
    assert L.semkv_append_decode(ref, nul, one, one, one, sc, one, one, 1 << 30, nul) == 1   # null k
    s.L_hi_v = 3  # a shape on the two-call path: the same checks come first
    assert L.semkv_append_decode(ref, one, one, one, nul, sc, one, one, 1 << 30, nul) == 1
    s.L_hi_v = 0
    assert semkv.status_string(3) == "SEMKV_ERR_CAPACITY"
    # the bounded-wait self-test: null status, test bound or use_tmem out of range
    assert L.semkv_selftest_wait_timeout(nul, 16, 1, nul) == 1
    assert L.semkv_selftest_wait_timeout(one, 0, 1, nul) == 1
    assert L.semkv_selftest_wait_timeout(one, (1 << 16) + 1, 1, nul) == 1
    assert L.semkv_selftest_wait_timeout(one, 16, 2, nul) == 1


@pytest.mark.parametrize("L_hi,L_lo,L_hi_v,L_lo_v", [(8, 5, 3, 2), (16, 8, 5, 4), (6, 4, 256, 17)])
def test_cache_bytes_with_v_levels_match_oracle_layout(semkv, orc, L_hi, L_lo, L_hi_v, L_lo_v):
    s = _shape(L_hi=L_hi, L_lo=L_lo, L_hi_v=L_hi_v, L_lo_v=L_lo_v)
    sizes = dict(zip(semkv._lib.BUF_NAMES, semkv.semkv_cache_bytes(s)))
    for seg, L, Lv, cap in (("hi", L_hi, L_hi_v, 256), ("lo", L_lo, L_lo_v, 768)):
        sh = orc.segment_shapes(128, 64, L, cap // 128, Lv)
        for name in ("k", "v", "kz", "vz"):
            n = 1
            for x in sh[name]:
                n *= x
            assert sizes[f"{name}_{seg}"] == 16 * n * 4, (seg, name)


def test_variant_fields_accept_their_ranges(semkv):
    for kw in (dict(window=0, clip=0.0), dict(window=10 ** 6, clip=1.0), dict(clip=1e-6), dict(clip=0.5)):
        assert len(semkv.semkv_cache_bytes(_shape(**kw))) == len(semkv._lib.BUF_NAMES)


def test_workspace_bytes_cover_the_split_partials(semkv):
    s = _shape()
    n = semkv.semkv_workspace_bytes(s)
    units, g, D = 16, 4, 128
    per_split = units * g * (D + 2) * 4
    assert n % per_split == 0 and 2 <= n // per_split <= 2 + 8  # at least one split per segment


def test_capacities_by_hand(semkv):
    """semkv_capacities: floor(p T) in double from the binary32 p, each segment rounded up to whole
    128-slot tiles, T_cap to whole 32-token bitmap words."""
    assert semkv.semkv_capacities(32768, 0.25) == (8192, 8192, 24576, 32768)
    assert semkv.semkv_capacities(32768, 0.25, extra=300) == (8192, 8576, 24960, 33088)
    assert semkv.semkv_capacities(1000, 0.3, window=16, extra=1) == (300, 384, 768, 1024)
    # 0.1 as binary32 is 0.100000001490116..., so floor(p * 10) = 1 (and not 0.99999...)
    assert semkv.semkv_capacities(10, 0.1)[0] == 1
    assert semkv.semkv_capacities(0, 0.5) == (0, 0, 0, 0)
    assert semkv.semkv_capacities(7, 1.0, window=100) == (7, 128, 0, 32)
    for bad in ((-1, 0.5, 0, 0), (10, 1.5, 0, 0), (10, -0.1, 0, 0), (10, 0.5, -1, 0), (10, 0.5, 0, -1),
                (2 ** 31 - 1, 0.5, 0, 2 ** 30)):
        with pytest.raises(semkv.SemkvError) as e:
            semkv.semkv_capacities(*bad)
        assert e.value.code == semkv._lib.SEMKV_ERR_INVALID_ARG, bad


def test_capacities_match_the_oracle_count(semkv, orc):
    import numpy as np

    r = np.random.default_rng(0)
    for _ in range(200):
        T = int(r.integers(0, 200000))
        p = float(np.float32(r.random()))
        assert semkv.semkv_capacities(T, p)[0] == orc.n_hi(p, T)
