"""Pins of the CPU oracle against what the SemKV page and the mathematics fix.

None of these re-types the oracle's formulas: each compares it with an independent routine
(numpy's IEEE binary16 conversion, Python's base-L integer parser, exact rational arithmetic,
brute-force enumeration, torch's scaled_dot_product_attention) or with an invariant of the
method (every token kept; p = 0 and p = 1 reduce to uniform quantization; bulk quantization and
token-by-token appends agree).
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- binary16


def test_half_to_float_matches_numpy_for_every_pattern(orc):
    h = np.arange(65536, dtype=np.uint16)
    f = orc.half_to_float(h)
    ref = h.view(np.float16).astype(np.float32)
    same = (f.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(f) & np.isnan(ref))
    assert same.all()


def _ru_numpy(x: np.ndarray) -> np.ndarray:
    """Round toward +inf to binary16, built from numpy's round-to-nearest conversion."""
    with np.errstate(over="ignore"):
        h = x.astype(np.float16)
        low = h.astype(np.float32) < x
        h[low] = np.nextafter(h[low], np.float16(np.inf))
    return h


def test_float_to_half_up_matches_numpy_round_up(orc):
    r = np.random.default_rng(1)
    parts = [
        r.standard_normal(200000).astype(np.float32) * np.float32(3.0),
        (r.standard_normal(50000) * 1e-5).astype(np.float32),  # subnormal range of binary16
        (r.standard_normal(50000) * 3e4).astype(np.float32),   # near the top of binary16
        np.array([0.0, 6e-8, 5.96e-8, 2 ** -24, 2 ** -25, 2 ** -14, 65504.0, 65504.5, 65519.0, 65520.0,
                  1e9, -1e9, -65504.5, 1.0 + 2 ** -11, 1.0 + 2 ** -12, -(1.0 + 2 ** -12)], np.float32),
    ]
    x = np.concatenate(parts)
    got = orc.float_to_half_up(x)
    ref = _ru_numpy(x).view(np.uint16)
    # numpy keeps -0 for tiny negatives rounded up; the oracle does the same
    assert np.array_equal(got, ref)


def test_scale_saturates_at_largest_finite_half(orc):
    assert orc.scale_half(70000.0) == 0x7BFF
    assert orc.scale_half(65504.0) == 0x7BFF
    assert orc.scale_half(0.0) == 0


# ---------------------------------------------------------------- radix packing


@pytest.mark.parametrize("L", range(2, 257))
def test_radix_digits_is_the_largest_power_in_32_bits(orc, L):
    k = orc.radix_digits(L)
    assert L ** k <= 2 ** 32 < L ** (k + 1)


def test_words_per_row_table_for_the_configured_levels(orc):
    # k(L) and words per 128-channel row for the level counts the workloads use
    table = {4: (16, 8), 5: (13, 10), 6: (12, 11), 8: (10, 13), 16: (8, 16)}
    for L, (k, W) in table.items():
        assert orc.radix_digits(L) == k
        assert orc.words_per_row(L, 128) == W
        assert orc.words_per_tile_column(L) == W  # tile of 128 slots = 128 channels


_DIG = "0123456789abcdefghijklmnopqrstuvwxyz"


@pytest.mark.parametrize("L", list(range(2, 37)))
def test_pack_is_base_L_positional_notation(orc, L):
    """word == int(digits, base=L) with the lowest-index code as the least significant digit."""
    k = orc.radix_digits(L)
    r = np.random.default_rng(L)
    for _ in range(200):
        c = r.integers(0, L, size=k).astype(np.uint8)
        c[r.integers(0, k)] = L - 1
        w = orc.pack_word(c, L)
        ref = int("".join(_DIG[int(d)] for d in c[::-1]), L)
        assert w == ref
        assert np.array_equal(orc.unpack_word(w, k, L), c)


def test_pack_power_of_two_levels_are_bit_fields(orc):
    r = np.random.default_rng(3)
    for L, bits in ((2, 1), (4, 2), (16, 4)):
        k = orc.radix_digits(L)
        assert k * bits == 32
        c = r.integers(0, L, size=k).astype(np.uint8)
        w = orc.pack_word(c, L)
        for i in range(k):
            assert (w >> (bits * i)) & (L - 1) == c[i]


def test_code_bits_printed_on_the_page(orc):
    page = json.load(open(os.path.join(GOLDEN, "page_values.json")))
    for e in page["code_bits"]:
        assert round(math.log2(e["levels"]), 3) == e["bits_printed"]
    lo, hi = page["cliff_interval_bits"]["lower_open"], page["cliff_interval_bits"]["upper_closed"]
    assert lo < math.log2(5) <= hi + 5e-4 and not (lo < math.log2(4))


# ---------------------------------------------------------------- select


def test_n_hi_is_floor_of_p_T_exactly(orc):
    r = np.random.default_rng(4)
    for _ in range(2000):
        p = np.float32(r.random())
        T = int(r.integers(0, 200000))
        assert orc.n_hi(p, T) == math.floor(Fraction(float(p)) * T)
    assert orc.n_hi(0.25, 32768) == 8192 and orc.n_hi(0.5, 131072) == 65536


def _brute_force_hi_set(scores, n):
    """Among all n-subsets: the largest exact score sum, then the lexicographically smallest
    sorted index list (lower token index wins among equal scores)."""
    best = None
    for sub in itertools.combinations(range(len(scores)), n):
        key = (sum(Fraction(float(scores[i])) for i in sub), [-i for i in sub])
        if best is None or key > best[0]:
            best = (key, sub)
    return set(best[1]) if best else set()


@pytest.mark.parametrize("seed", range(40))
def test_select_matches_brute_force_on_tiny_units(orc, seed):
    r = np.random.default_rng(seed)
    T = int(r.integers(1, 11))
    # few distinct values -> many ties; include both signed zeros
    vals = np.array([-1.5, -0.0, 0.0, 0.25, 2.0, 2.0], np.float32)
    scores = vals[r.integers(0, len(vals), size=T)]
    p = np.float32(r.integers(0, 9) / 8)
    bitmap, rank, n_hi, tau, st = orc.select(scores, p)
    assert st == 0
    want = _brute_force_hi_set(scores, math.floor(Fraction(float(p)) * T))
    got = {t for t in range(T) if (int(bitmap[t // 32]) >> (t % 32)) & 1}
    assert got == want
    assert n_hi == len(want)
    if n_hi:
        assert tau == np.sort(scores)[::-1][n_hi - 1]
        assert not (tau == 0 and np.signbit(tau))  # a zero threshold is stored as +0
    else:
        assert tau == np.inf


def test_select_every_token_kept_and_rank_is_prefix_popcount(orc):
    r = np.random.default_rng(5)
    for T in (1, 31, 32, 33, 4095, 5000):
        scores = r.standard_normal(T).astype(np.float32)
        for p in (0.0, 0.25, 0.5, 1.0):
            bitmap, rank, n_hi, tau, st = orc.select(scores, p)
            ones = [bin(int(w)).count("1") for w in bitmap]
            assert sum(ones) == n_hi
            assert n_hi + (T - n_hi) == T
            assert list(rank) == [sum(ones[:w]) for w in range(len(ones))]
            tail = T % 32
            if tail:
                assert int(bitmap[-1]) >> tail == 0  # no bits past the last token
            if p == 0.0:
                assert n_hi == 0 and not bitmap.any() and tau == np.inf
            if p == 1.0:
                assert n_hi == T and tau == scores.min()


def test_select_flags_nan(orc):
    s = np.array([1.0, np.nan, 2.0], np.float32)
    assert orc.select(s, 0.5)[4] & orc.NAN_SCORE


# ---------------------------------------------------------------- quantize


def _grid(orc, x16, L):
    codes, s16, z16, st = orc.quantize_group(x16, L)
    s = float(np.uint16(s16).view(np.float16))
    z = float(np.uint16(z16).view(np.float16))
    return codes, s, z, st


@pytest.mark.parametrize("L", [2, 3, 4, 5, 6, 7, 8, 16, 31, 256])
def test_values_on_the_grid_round_trip_exactly(orc, L):
    r = np.random.default_rng(L)
    for G in (32, 64, 128):
        for e in (-6, -2, 0, 3):
            s = 2.0 ** e
            z = float(r.integers(-8, 8)) * s
            c = r.integers(0, L, size=G)
            c[0], c[-1] = 0, L - 1
            x = (z + c * s).astype(np.float16)
            assert np.array_equal(x.astype(np.float64), z + c * s)  # exactly representable
            codes, s_got, z_got, st = _grid(orc, x.view(np.uint16), L)
            assert st == 0
            assert s_got == s and z_got == z
            assert np.array_equal(codes, c)


def _exact_nearest(x, s, z, L):
    cand = z + np.arange(L)[None, :] * s
    return np.abs(x[:, None] - cand)


@pytest.mark.parametrize("L", [3, 4, 5, 6, 8, 16])
def test_quantizer_is_nearest_grid_point_and_within_half_step(orc, L):
    r = np.random.default_rng(10 + L)
    for trial in range(300):
        G = (32, 64, 128)[trial % 3]
        x = (r.standard_normal(G) * 10 ** r.uniform(-3, 3)).astype(np.float16)
        codes, s, z, st = _grid(orc, x.view(np.uint16), L)
        xf = x.astype(np.float64)
        assert codes.max() <= L - 1
        assert codes[np.argmin(xf)] == 0 and codes[np.argmax(xf)] == L - 1
        # scale: the smallest binary16 >= the fp32 quotient (numpy fp32 arithmetic, RN)
        sf = (np.float32(xf.max()) - np.float32(xf.min())) / np.float32(L - 1)
        assert s == float(_ru_numpy(np.array([sf], np.float32))[0])
        assert z == xf.min()
        # monotone in x
        o = np.argsort(xf, kind="stable")
        assert np.all(np.diff(codes[o].astype(int)) >= 0)
        # nearest grid point, up to fp32 rounding of (x - z)/s at exact half-steps
        dist = _exact_nearest(xf, s, z, L)
        mine = dist[np.arange(G), codes]
        assert np.all(mine <= dist.min(axis=1) + s * 2 ** -20)
        # |x - x^| <= s/2 (+ fp32 rounding of the fma and of (x - z)/s)
        # fmaf(c, s, z): the product and sum are exact in float64 here; one rounding to fp32
        xh = (codes.astype(np.float64) * s + z).astype(np.float32).astype(np.float64)
        tol = s / 2 + 4 * np.spacing(np.float32(np.abs(xf).max()))
        assert np.all(np.abs(xf - xh) <= tol)


def test_constant_group_gives_zero_scale_and_exact_values(orc):
    for v in (0.0, -0.0, 1.5, -3.25, 65504.0):
        x = np.full(64, v, np.float16)
        codes, s, z, st = _grid(orc, x.view(np.uint16), 5)
        assert s == 0.0 and not codes.any() and z == v
        assert np.uint16(orc.quantize_group(x.view(np.uint16), 5)[2]) != 0x8000  # -0 stored as +0


def test_nonfinite_values_are_flagged(orc):
    x = np.zeros(32, np.float16)
    x[3] = np.inf
    assert orc.quantize_group(x.view(np.uint16), 5)[3] & orc.NONFINITE_KV
    x[3] = np.nan
    assert orc.quantize_group(x.view(np.uint16), 5)[3] & orc.NONFINITE_KV


# ---------------------------------------------------------------- unit: place, storage, uniform limits


def _unit(orc, T, D, G, L_hi, L_lo, p, seed):
    r = np.random.default_rng(seed)
    K = r.standard_normal((T, D)).astype(np.float16)
    V = r.standard_normal((T, D)).astype(np.float16)
    sc = r.standard_normal(T).astype(np.float32)
    bm, rk, nh, tau, st = orc.select(sc, p)
    th = max(1, -(-nh // 128))
    tl = max(1, -(-(T - nh) // 128))
    hi, lo, st2 = orc.quantize_pack_unit(K.view(np.uint16), V.view(np.uint16), bm, G, L_hi, L_lo, th, tl)
    return dict(K=K, V=V, sc=sc, bm=bm, rk=rk, nh=nh, tau=tau, hi=hi, lo=lo, st=st | st2, th=th, tl=tl)


def test_every_token_is_kept_and_dequantizes_within_half_step(orc):
    u = _unit(orc, 300, 128, 64, 8, 5, 0.25, 0)
    assert u["st"] == 0
    Kh, Vh = orc.dequantize_unit(300, 128, 64, 8, 5, u["bm"], u["hi"], u["lo"])
    assert Kh.shape == (300, 128)
    for X, Xh in ((u["K"], Kh), (u["V"], Vh)):
        xf = X.astype(np.float64).reshape(300, 2, 64)
        rng = xf.max(-1) - xf.min(-1)
        for t in range(300):
            L = 8 if (int(u["bm"][t // 32]) >> (t % 32)) & 1 else 5
            bound = rng[t] / (L - 1) * (1 + 2 ** -10) / 2 + 1e-6
            assert np.all(np.abs(xf[t] - Xh[t].reshape(2, 64)) <= bound[:, None])


@pytest.mark.parametrize("L", [4, 5, 6, 8, 16])
def test_p0_and_p1_reduce_to_uniform_quantization(orc, L):
    r = np.random.default_rng(L)
    T, D, G = 260, 128, 32
    K = r.standard_normal((T, D)).astype(np.float16).view(np.uint16)
    V = r.standard_normal((T, D)).astype(np.float16).view(np.uint16)
    sc = r.standard_normal(T).astype(np.float32)
    bm1 = orc.select(sc, 1.0)[0]
    bm0 = orc.select(sc, 0.0)[0]
    hi1, _, _ = orc.quantize_pack_unit(K, V, bm1, G, L, 3, 3, 1)
    _, lo0, _ = orc.quantize_pack_unit(K, V, bm0, G, 7, L, 1, 3)
    for name in ("k", "v", "kz", "vz"):
        assert np.array_equal(hi1[name], lo0[name])


def test_average_code_bits_interpolate_between_the_two_grids(orc):
    """Mixing two grids reaches an average precision between them (page: grid interpolation)."""
    for (L_hi, L_lo) in ((6, 5), (8, 5), (8, 6), (16, 8)):
        for p in (0.0, 0.25, 0.5, 0.75, 1.0):
            T = 4096
            u = _unit(orc, T, 128, 128, L_hi, L_lo, p, 7)
            p_real = u["nh"] / T
            ideal = p_real * math.log2(L_hi) + (1 - p_real) * math.log2(L_lo)
            # packed bits per code actually used: words of each segment x 32 / (tokens x 128)
            k_bits = (32 * u["hi"]["k"].shape[1] * u["nh"] + 32 * u["lo"]["k"].shape[1] * (T - u["nh"])) / (T * 128)
            assert math.log2(L_lo) - 1e-12 <= ideal <= math.log2(L_hi) + 1e-12
            assert ideal <= k_bits  # packing never beats the entropy of the grid
            assert k_bits <= ideal + 0.5  # one 32-bit word holds floor(32 / log2 L) codes at least


def test_storage_ratio_closed_form_matches_buffer_bytes(orc):
    """bits/value = [p*32*W(L_hi) + (1-p)*32*W(L_lo)]/D + 32/G + 1/(2D) equals the bytes the
    oracle's buffers take for full tiles, counted independently here."""
    for (L_hi, L_lo) in ((6, 5), (8, 6), (16, 8)):
        for G in (32, 64, 128):
            for p in (0.0, 0.25, 0.5, 0.75, 1.0):
                T = 128 * 16
                nh = math.floor(p * T)
                hi = orc.segment_shapes(128, G, L_hi, nh // 128)
                lo = orc.segment_shapes(128, G, L_lo, (T - nh) // 128)
                words = sum(int(np.prod(s)) for s in hi.values()) + sum(int(np.prod(s)) for s in lo.values())
                bits = (words * 32 + T) / (2 * T * 128)  # K and V values, plus the 1-bit bitmap
                W = {L: math.ceil(128 / orc.radix_digits(L)) for L in (L_hi, L_lo)}
                closed = (p * 32 * W[L_hi] + (1 - p) * 32 * W[L_lo]) / 128 + 32 / G + 1 / 256
                assert abs(bits - closed) < 1e-12
                assert abs(orc.storage_bits_per_value(128, G, L_hi, L_lo, p) - closed) < 1e-12


def test_quantize_pack_flags_nonfinite_input(orc):
    r = np.random.default_rng(0)
    K = r.standard_normal((40, 128)).astype(np.float16)
    V = r.standard_normal((40, 128)).astype(np.float16)
    V[7, 3] = np.inf
    bm = orc.select(r.standard_normal(40).astype(np.float32), 0.5)[0]
    _, _, st = orc.quantize_pack_unit(K.view(np.uint16), V.view(np.uint16), bm, 64, 8, 5, 1, 1)
    assert st & orc.NONFINITE_KV


# ---------------------------------------------------------------- append


@pytest.mark.parametrize("p,L", [(0.0, 5), (1.0, 6)])
def test_appending_tokens_equals_quantizing_them_in_bulk(orc, p, L):
    """With p = 0 (tau = +inf: every new token goes lo) or p = 1 (new tokens above the smallest
    prefill score go hi), appending tokens one at a time must give the same bytes as quantizing
    the whole sequence at once."""
    r = np.random.default_rng(11)
    T0, T, D, G = 150, 300, 128, 64
    K = r.standard_normal((T, D)).astype(np.float16).view(np.uint16)
    V = r.standard_normal((T, D)).astype(np.float16).view(np.uint16)
    sc = r.standard_normal(T).astype(np.float32)
    sc[T0:] = 100.0  # above every prefill score
    tiles = 3
    bm, rk, nh, tau, _ = orc.select(sc, p)
    hiA, loA, _ = orc.quantize_pack_unit(K, V, bm, G, L, L, tiles, tiles)
    bm0, rk0, nh0, tau0, _ = orc.select(sc[:T0], p)
    hi0, lo0, _ = orc.quantize_pack_unit(K[:T0], V[:T0], bm0, G, L, L, tiles, tiles)
    st = orc.UnitState(512, bm0, rk0, nh0, T0 - nh0, tau0, hi0, lo0)
    for t in range(T0, T):
        assert orc.append_unit(st, K[t], V[t], sc[t], G, L, L) == 0
    assert st.n_hi + st.n_lo == T
    nw = (T + 31) // 32
    assert np.array_equal(st.bitmap[:nw], bm) and np.array_equal(st.rank[:nw], rk)
    for name in ("k", "v", "kz", "vz"):
        assert np.array_equal(st.hi[name], hiA[name])
        assert np.array_equal(st.lo[name], loA[name])


def test_append_decision_and_capacity(orc):
    r = np.random.default_rng(12)
    T0, D, G = 64, 128, 128
    K = r.standard_normal((T0 + 4, D)).astype(np.float16).view(np.uint16)
    sc = r.standard_normal(T0).astype(np.float32)
    bm, rk, nh, tau, _ = orc.select(sc, 0.25)
    hi, lo, _ = orc.quantize_pack_unit(K[:T0], K[:T0], bm, G, 8, 5, 1, 1)
    st = orc.UnitState(128, bm, rk, nh, T0 - nh, tau, hi, lo)
    # equal to tau -> lo (strict), above -> hi
    assert orc.append_unit(st, K[T0], K[T0], float(tau), G, 8, 5) == 0
    assert (int(st.bitmap[T0 // 32]) >> (T0 % 32)) & 1 == 0
    assert orc.append_unit(st, K[T0 + 1], K[T0 + 1], float(tau) + 1.0, G, 8, 5) == 0
    assert (int(st.bitmap[(T0 + 1) // 32]) >> ((T0 + 1) % 32)) & 1 == 1
    # fill the hi segment (one tile) and overflow it
    while st.n_hi < 128:
        assert orc.append_unit(st, K[T0], K[T0], 1e9, G, 8, 5) == 0 or st.n_hi + st.n_lo >= 128
        if st.n_hi + st.n_lo >= 128:
            break
    assert orc.append_unit(st, K[T0], K[T0], 1e9, G, 8, 5) & orc.OVERFLOW


# ---------------------------------------------------------------- attention


def _sdpa_fp64(q16, Kh, Vh, scale):
    import torch

    q = torch.from_numpy(q16.astype(np.float64))[None, :, None, :]  # [1, g, 1, D]
    k = torch.from_numpy(Kh.astype(np.float64))[None, None].expand(1, q.shape[1], -1, -1)
    v = torch.from_numpy(Vh.astype(np.float64))[None, None].expand(1, q.shape[1], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale)
    return o[0, :, 0].numpy()


@pytest.mark.parametrize("T,g", [(1, 4), (7, 1), (100, 4), (513, 8)])
def test_attention_matches_torch_sdpa_in_fp64(orc, T, g):
    r = np.random.default_rng(T)
    D = 128
    q = r.standard_normal((g, D)).astype(np.float16)
    Kh = (r.standard_normal((T, D)) * 2).astype(np.float32)
    Vh = r.standard_normal((T, D)).astype(np.float32)
    got = orc.attention_fp64(q.view(np.uint16), Kh, Vh, 1 / math.sqrt(D))
    ref = _sdpa_fp64(q, Kh, Vh, float(np.float32(1 / math.sqrt(D))))
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_attention_one_hot_and_uniform_logits(orc):
    D, T = 128, 50
    r = np.random.default_rng(0)
    Vh = r.standard_normal((T, D)).astype(np.float32)
    q = np.zeros((1, D), np.float16)
    q[0, 0] = 1.0
    Kh = np.zeros((T, D), np.float32)
    Kh[17, 0] = 1e4  # one logit far above the rest
    o = orc.attention_fp64(q.view(np.uint16), Kh, Vh, 1.0)
    assert np.allclose(o[0], Vh[17], atol=1e-12)
    o = orc.attention_fp64(q.view(np.uint16), np.zeros((T, D), np.float32), Vh, 1.0)
    assert np.allclose(o[0], Vh.astype(np.float64).mean(0), atol=1e-12)
    o = orc.attention_fp64(q.view(np.uint16), np.zeros((0, D), np.float32), np.zeros((0, D), np.float32), 1.0)
    assert not o.any()


@pytest.mark.parametrize("T,g", [(1, 4), (100, 4), (513, 8), (4096, 4)])
def test_attention_f32_matches_torch_sdpa_in_fp32(orc, T, g):
    """The fp32-accumulate attention (the timed CPU variant) against torch's fp32 SDPA, within the
    rounding of binary32 sums over T terms."""
    import torch

    r = np.random.default_rng(T + 1)
    D = 128
    q = r.standard_normal((g, D)).astype(np.float16)
    Kh = (r.standard_normal((T, D)) * 2).astype(np.float32)
    Vh = r.standard_normal((T, D)).astype(np.float32)
    got = orc.attention_f32(q.view(np.uint16), Kh, Vh, float(np.float32(1 / math.sqrt(D))))
    assert got.dtype == np.float32
    qt = torch.from_numpy(q.astype(np.float32))[None, :, None, :]
    kt = torch.from_numpy(Kh)[None, None].expand(1, g, -1, -1)
    vt = torch.from_numpy(Vh)[None, None].expand(1, g, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=float(np.float32(1 / math.sqrt(D))))
    assert np.allclose(got, ref[0, :, 0].numpy(), rtol=1e-4, atol=2e-5)


def test_attention_f32_one_hot_uniform_and_empty(orc):
    D, T = 128, 50
    r = np.random.default_rng(2)
    Vh = r.standard_normal((T, D)).astype(np.float32)
    q = np.zeros((1, D), np.float16)
    q[0, 0] = 1.0
    Kh = np.zeros((T, D), np.float32)
    Kh[17, 0] = 1e4
    assert np.array_equal(orc.attention_f32(q.view(np.uint16), Kh, Vh, 1.0)[0], Vh[17])
    o = orc.attention_f32(q.view(np.uint16), np.zeros((T, D), np.float32), Vh, 1.0)
    assert np.allclose(o[0], Vh.astype(np.float64).mean(0), atol=1e-6)
    o = orc.attention_f32(q.view(np.uint16), np.zeros((0, D), np.float32), np.zeros((0, D), np.float32), 1.0)
    assert not o.any()


def test_layout_as_documented(orc):
    """Read the oracle's buffers with plain indexing per the documented layout and check each
    digit against a one-group quantization of that token's row (K: row words; V: column words)."""
    T, D, G, L_hi, L_lo = 300, 128, 64, 8, 5
    u = _unit(orc, T, D, G, L_hi, L_lo, 0.25, 3)
    slot = {0: 0, 1: 0}
    for t in range(T):
        seg = 0 if (int(u["bm"][t // 32]) >> (t % 32)) & 1 else 1
        s = slot[seg]
        slot[seg] += 1
        buf = u["hi"] if seg == 0 else u["lo"]
        L = L_hi if seg == 0 else L_lo
        k = orc.radix_digits(L)
        tile, tt = divmod(s, 128)
        for X, name in ((u["K"], "k"), (u["V"], "v")):
            for grp in range(D // G):
                codes, s16, z16, _ = orc.quantize_group(X[t, grp * G:(grp + 1) * G].view(np.uint16), L)
                assert buf[name + "z"][tile, grp, tt] == s16 | (z16 << 16)
                for i, c in enumerate(codes):
                    d = grp * G + i
                    if name == "k":
                        w = int(buf["k"][tile, d // k, tt])
                        digit = d % k
                    else:
                        w = int(buf["v"][tile, tt // k, d])
                        digit = tt % k
                    assert (w // L ** digit) % L == c
