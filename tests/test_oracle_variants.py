"""Pins of the oracle's quantizer variants (prior art summarised on the same pages, the SKVQ
abstract: clipped dynamic group quantization; the most recent tokens kept at high precision).

The clipped grid [reading]: mn' = clip*mn, mx' = clip*mx (fp32); z = nearest binary16 of mn'
(ties to even, -0 stored as +0); s = binary16 rounded up of (mx' - z)/(L - 1), at least 0; codes
clamp(rint((x - z)/s), 0, L - 1).  The window [reading]: after the selection by score the last
min(W, T) tokens go to the finer grid too; n_hi counts them; tau is the score threshold.
Expected values below are worked out by hand from those definitions, or are brute force."""
import numpy as np
import pytest

import oracle


def h16(vals):
    return np.array(vals, dtype=np.float16).view(np.uint16)


def test_clip_worked_example_exact_grid():
    # range [-2, 2] at clip 0.5 -> [-1, 1]; L = 5: z = -1, s = 2/4 = 0.5 (both exact)
    x = h16([-2, -1, 0, 1, 2, 0.25, -0.75, 1.5])
    c, s16, z16, st = oracle.quantize_group(x, 5, clip=0.5)
    assert st == 0
    assert s16 == 0x3800 and z16 == 0xBC00  # 0.5 and -1.0
    # (x + 1)/0.5 = -2, 0, 2, 4, 6, 2.5, 0.5, 5 -> rint (ties to even), clamp to [0, 4]
    assert c.tolist() == [0, 0, 2, 4, 4, 2, 0, 4]


def test_clip_worked_example_rounded_zero():
    # clip 0.3 of [-1, 1]: mn' = -0.300000011920928955078125 (the fp32 0.3).  Binary16 spacing in
    # [0.25, 0.5) is 2^-12: 0.3000000119 / 2^-12 = 1228.80005 -> 1229 -> z = -0.300048828125 = 0xB4CD.
    # mx' - z = 0.600048840045928955078125 (exact in fp32: 10067149 * 2^-24); / 4 = 0.15001221..;
    # rounded up on the 2^-13 spacing of [0.125, 0.25): 1228.9 -> 1229 -> s = 0.1500244140625 = 0x30CD.
    x = h16([-1, 1, 0, 0.25, -0.125])
    c, s16, z16, st = oracle.quantize_group(x, 5, clip=0.3)
    assert (s16, z16) == (0x30CD, 0xB4CD)
    # (x - z)/s: -4.67 -> 0; 8.67 -> 4; exactly 2 (z = 2 s); 3.67 -> 4; 1.167 -> 1
    assert c.tolist() == [0, 4, 2, 4, 1]


def test_half_rn_ties_and_range():
    assert oracle.half_rn(1.0) == 0x3C00
    assert oracle.half_rn(1.0 + 2.0 ** -11) == 0x3C00          # tie between 1 and 1 + 2^-10: even
    assert oracle.half_rn(1.0 + 3 * 2.0 ** -11) == 0x3C02      # tie between 1+2^-10 and 1+2^-9: even
    assert oracle.half_rn(1.0 + 2.0 ** -11 + 2.0 ** -20) == 0x3C01
    assert oracle.half_rn(-2.0 ** -25) == 0x8000               # half the smallest subnormal: tie to 0
    assert oracle.half_rn(-3 * 2.0 ** -26) == 0x8001           # 0.75 of it: nearest is the subnormal
    assert oracle.half_rn(65504.0) == 0x7BFF and oracle.half_rn(65519.0) == 0x7BFF
    assert oracle.half_rn(65520.0) == 0x7C00


def test_clip_negative_zero_and_constant_group():
    # smallest negative subnormal and 0 at clip 0.25: mn' = -2^-26 rounds to -0, stored as +0
    c, s16, z16, _ = oracle.quantize_group(np.array([0x8001, 0x0000], np.uint16), 4, clip=0.25)
    assert z16 == 0x0000 and s16 == 0x0000 and c.tolist() == [0, 0]
    # constant group 3.0 at clip 0.7: z = rn16(fp32(0.7) * 3) = rn16(2.1000001) on spacing 2^-9:
    # 1075.2 -> 1075 -> 2.099609375 = 0x4033; (mx' - z) > 0 so s = ru16((2.1000001 - 2.0996094)/L-1)
    c, s16, z16, _ = oracle.quantize_group(h16([3.0] * 4), 3, clip=0.7)
    assert z16 == 0x4033
    assert c.tolist() == [2, 2, 2, 2]  # 3 is far above the clipped range: top code


@pytest.mark.parametrize("clip,L", [(0.9, 5), (0.6, 8), (0.35, 16), (0.75, 2)])
def test_clip_error_bound_property(clip, L):
    """Inside the clipped grid every value is within s/2 (plus fp32 rounding) of its dequantized
    value; below it the code is 0, above it L - 1."""
    r = np.random.default_rng(int(clip * 100) + L)
    for _ in range(200):
        x = (r.standard_normal(64) * r.choice([0.01, 1, 50])).astype(np.float16)
        c, s16, z16, st = oracle.quantize_group(x.view(np.uint16), L, clip=clip)
        assert st == 0
        s = float(np.uint16(s16).view(np.float16))
        z = float(np.uint16(z16).view(np.float16))
        xf = x.astype(np.float64)
        top = z + (L - 1) * s
        assert top >= clip * float(xf.max()) - 1e-12  # the grid reaches the clipped maximum
        xhat = c.astype(np.float64) * s + z  # the grid point, exactly (float64 holds it)
        inside = (xf >= z) & (xf <= top)
        tol = s / 2 + 4 * np.finfo(np.float32).eps * (abs(z) + (L - 1) * s)
        assert np.all(np.abs(xhat[inside] - xf[inside]) <= tol)
        assert np.all(c[xf < z] == 0)
        assert np.all(c[xf > top] == L - 1)
        assert np.all(c <= L - 1)


def test_clip_one_is_the_plain_grid():
    r = np.random.default_rng(3)
    for _ in range(100):
        x = r.standard_normal(32).astype(np.float16).view(np.uint16)
        a = oracle.quantize_group(x, 6)
        b = oracle.quantize_group(x, 6, clip=1.0)
        assert a[0].tolist() == b[0].tolist() and a[1:] == b[1:]


def _brute_select(score, p, W):
    T = len(score)
    n = int(np.floor(float(np.float32(p)) * T))
    key = lambda t: (-(float(score[t]) + 0.0), t)  # noqa: E731  (-0 == +0; lower index first)
    order = sorted(range(T), key=key)
    hi = set(order[:n]) | set(range(max(T - W, 0), T))
    tau = float(score[order[n - 1]]) + 0.0 if n > 0 else np.inf
    return hi, tau


@pytest.mark.parametrize("T,p,W", [(1, 0.0, 1), (37, 0.25, 5), (100, 0.5, 0), (100, 0.1, 100), (65, 0.3, 200),
                                   (64, 0.0, 7), (200, 1.0, 13)])
def test_window_select_brute_force(T, p, W):
    r = np.random.default_rng(T + W)
    score = r.integers(-5, 5, T).astype(np.float32)  # many ties
    score[r.random(T) < 0.1] = -0.0
    bm, rk, nh, tau, st = oracle.select(score, p, window=W)
    hi, tau_ref = _brute_select(score, p, W)
    got = {t for t in range(T) if (int(bm[t // 32]) >> (t % 32)) & 1}
    assert got == hi
    assert nh == len(hi)
    assert float(tau) == tau_ref
    for w in range(len(rk)):
        assert rk[w] == sum(1 for t in hi if t < 32 * w)


def test_window_zero_is_plain_selection():
    r = np.random.default_rng(9)
    s = r.standard_normal(300).astype(np.float32)
    a = oracle.select(s, 0.3)
    b = oracle.select(s, 0.3, window=0)
    assert all(np.array_equal(np.asarray(x), np.asarray(y)) for x, y in zip(a, b))
    assert oracle.select(s, 0.3, window=-1)[4] == oracle.BAD_ARG


def test_clipped_unit_matches_its_groups():
    """quantize_pack_unit with a clip places, per token and group, the clipped group's codes."""
    r = np.random.default_rng(4)
    T, D, G = 150, 128, 32
    K = r.standard_normal((T, D)).astype(np.float16).view(np.uint16)
    V = r.standard_normal((T, D)).astype(np.float16).view(np.uint16)
    bm, _, nh, _, _ = oracle.select(r.standard_normal(T).astype(np.float32), 0.3)
    hi, lo, st = oracle.quantize_pack_unit(K, V, bm, G, 8, 5, 1, 2, clip=0.8)
    assert st == 0
    Kh, Vh = oracle.dequantize_unit(T, D, G, 8, 5, bm, hi, lo)
    for t in (0, 77, 149):
        is_hi = (int(bm[t // 32]) >> (t % 32)) & 1
        L = 8 if is_hi else 5
        for g in range(D // G):
            c, s16, z16, _ = oracle.quantize_group(K[t, g * G:(g + 1) * G], L, clip=0.8)
            s = np.uint16(s16).view(np.float16).astype(np.float32)
            z = np.uint16(z16).view(np.float16).astype(np.float32)
            ref = (c.astype(np.float32) * s).astype(np.float32) + z
            assert np.allclose(Kh[t, g * G:(g + 1) * G], ref, rtol=0, atol=1e-6 * (1 + abs(float(z))))


# ---------------------------------------------------------------- separate V level counts


def _digits(w, L, k):
    out = []
    for _ in range(k):
        w, d = divmod(int(w), L)
        out.append(d)
    return out


def test_separate_v_levels_words_decode_by_hand():
    """K words in base L_k, V words in base L_v: decoded here with divmod, the codes are those
    of each token's groups quantized on the tensor's own level count."""
    r = np.random.default_rng(12)
    T, D, G, Lh, Ll, Lhv, Llv = 70, 128, 32, 8, 5, 3, 2
    K = r.standard_normal((T, D)).astype(np.float16).view(np.uint16)
    V = r.standard_normal((T, D)).astype(np.float16).view(np.uint16)
    bm, _, nh, _, _ = oracle.select(r.standard_normal(T).astype(np.float32), 0.4)
    hi, lo, st = oracle.quantize_pack_unit(K, V, bm, G, Lh, Ll, 1, 1, L_hi_v=Lhv, L_lo_v=Llv)
    assert st == 0
    assert hi["v"].shape == (1, -(-128 // 20), D) and lo["v"].shape == (1, 4, D)  # k(3) = 20, k(2) = 32
    slots = {0: 0, 1: 0}
    for t in range(T):
        is_hi = (int(bm[t // 32]) >> (t % 32)) & 1
        seg, Lk, Lv = (hi, Lh, Lhv) if is_hi else (lo, Ll, Llv)
        slot = slots[is_hi]
        slots[is_hi] += 1
        kk, kv = oracle.radix_digits(Lk), oracle.radix_digits(Lv)
        kc = sum((_digits(seg["k"][0, j, slot], Lk, kk) for j in range(seg["k"].shape[1])), [])[:D]
        vc = [_digits(seg["v"][0, slot // kv, d], Lv, kv)[slot % kv] for d in range(D)]
        for g in range(D // G):
            ck = oracle.quantize_group(K[t, g * G:(g + 1) * G], Lk)[0]
            cv = oracle.quantize_group(V[t, g * G:(g + 1) * G], Lv)[0]
            assert kc[g * G:(g + 1) * G] == ck.tolist()
            assert vc[g * G:(g + 1) * G] == cv.tolist()


def test_separate_v_levels_equal_counts_are_the_default():
    r = np.random.default_rng(13)
    K = r.standard_normal((150, 128)).astype(np.float16).view(np.uint16)
    V = r.standard_normal((150, 128)).astype(np.float16).view(np.uint16)
    bm, _, _, _, _ = oracle.select(r.standard_normal(150).astype(np.float32), 0.3)
    a = oracle.quantize_pack_unit(K, V, bm, 64, 8, 5, 1, 1)
    b = oracle.quantize_pack_unit(K, V, bm, 64, 8, 5, 1, 1, L_hi_v=8, L_lo_v=5)
    for seg in (0, 1):
        for n in a[seg]:
            assert np.array_equal(a[seg][n], b[seg][n])


def test_separate_v_levels_storage_by_hand():
    # D 128, G 64.  hi: K L=8 (10 digits/word -> 13 words per row), V L=3 (20 -> 7 words per
    # 128-slot column); lo: K L=5 (13 -> 10), V L=2 (32 -> 4).  Per value, K and V averaged, plus
    # 32 bits of scale/zero per group of 64: hi (13 + 7)/2 * 32/128 + 0.5 = 3.0; lo (10 + 4)/2 *
    # 32/128 + 0.5 = 2.25.  p = 0.25, and the bitmap's 1/256: 0.75 + 1.6875 + 0.00390625.
    assert oracle.storage_bits_per_value(128, 64, 8, 5, 0.25, 3, 2) == pytest.approx(2.44140625, abs=1e-12)
    assert oracle.storage_bits_per_value(128, 64, 8, 5, 0.25, 8, 5) == oracle.storage_bits_per_value(128, 64, 8, 5,
                                                                                                    0.25)


def test_separate_v_levels_appends_equal_a_prefill():
    """Appending tokens one at a time leaves the same buffers as packing them all at once with the
    same assignment (both with the separate V levels and a clip)."""
    r = np.random.default_rng(14)
    T0, T, D, G, Lh, Ll, Lhv, Llv, clip = 100, 180, 128, 64, 6, 4, 3, 2, 0.8
    K = r.standard_normal((T, D)).astype(np.float16).view(np.uint16)
    V = r.standard_normal((T, D)).astype(np.float16).view(np.uint16)
    S = r.standard_normal(T).astype(np.float32)
    bm, rk, nh, tau, _ = oracle.select(S[:T0], 0.3)
    hi, lo, _ = oracle.quantize_pack_unit(K[:T0], V[:T0], bm, G, Lh, Ll, 2, 2, clip=clip, L_hi_v=Lhv, L_lo_v=Llv)
    st = oracle.UnitState(256, bm, rk, nh, T0 - nh, tau, hi, lo)
    for t in range(T0, T):
        assert oracle.append_unit(st, K[t], V[t], S[t], G, Lh, Ll, clip, Lhv, Llv) == 0
    hi2, lo2, _ = oracle.quantize_pack_unit(K, V, st.bitmap[:(T + 31) // 32], G, Lh, Ll, 2, 2, clip=clip,
                                            L_hi_v=Lhv, L_lo_v=Llv)
    for a, b in ((st.hi, hi2), (st.lo, lo2)):
        for n in a:
            assert np.array_equal(a[n], b[n]), n


# ---------------------------------------------------------------- per-channel K grids


def test_k_channel_grid_worked_by_hand():
    """Channel 0 holds -1, 0, 1, 2 over four tokens (the other channels 0).  Its hi grid (L 5) is
    s = 3/4 = 0.75 (exact), z = -1; its lo grid (L 3) s = 1.5, z = -1.  Tokens 0, 2 on hi and 1, 3
    on lo: codes 0 ((-1+1)/0.75), 1 ((0+1)/1.5 = 0.67), 3 ((1+1)/0.75 = 2.67), 2 ((2+1)/1.5)
    -> dequantized -1, 0.5, 1.25, 2.  Constant channels get s = 0, z = 0."""
    T, D = 4, 128
    K = np.zeros((T, D), np.float16)
    K[:, 0] = [-1, 0, 1, 2]
    K16 = K.view(np.uint16)
    kc, st = oracle.k_channel_grid(K16, 5, 3)
    assert st == 0
    assert kc[0, 0] == (0x3A00 | (0xBC00 << 16))  # 0.75 | -1.0
    assert kc[1, 0] == (0x3E00 | (0xBC00 << 16))  # 1.5 | -1.0
    assert (kc[:, 1:] == 0).all()
    bm = np.array([0b0101], np.uint32)
    V = np.zeros((T, D), np.float16).view(np.uint16)
    hi, lo, st = oracle.quantize_pack_unit(K16, V, bm, 64, 5, 3, 1, 1, kc=kc)
    assert st == 0
    assert not hi["kz"].any() and not lo["kz"].any()  # no per-token K grids in this mode
    Kh, _ = oracle.dequantize_unit(T, D, 64, 5, 3, bm, hi, lo, kc=kc)
    assert Kh[:, 0].tolist() == [-1.0, 0.5, 1.25, 2.0]
    assert not Kh[:, 1:].any()


def test_k_channel_grid_appends_clamp_to_the_prefill_grid():
    T, D = 4, 128
    K = np.zeros((T, D), np.float16)
    K[:, 0] = [-1, 0, 1, 2]
    kc, _ = oracle.k_channel_grid(K.view(np.uint16), 5, 3)
    bm, rk, nh, tau, _ = oracle.select(np.float32([3, 0, 2, 1]), 0.5)  # tokens 0, 2 hi; tau = 2
    hi, lo, _ = oracle.quantize_pack_unit(K.view(np.uint16), np.zeros((T, D), np.uint16), bm, 64, 5, 3, 1, 1, kc=kc)
    st = oracle.UnitState(32, bm, rk, nh, T - nh, tau, hi, lo, kc=kc)
    for x, score in ((5.0, 9.0), (-3.0, 9.0), (0.4, -9.0)):  # hi, hi, lo
        k = np.zeros(D, np.float16)
        k[0] = x
        assert oracle.append_unit(st, k.view(np.uint16), np.zeros(D, np.uint16), score, 64, 5, 3) == 0
    Kh, _ = oracle.dequantize_unit(T + 3, D, 64, 5, 3, st.bitmap, st.hi, st.lo, kc=kc)
    # 5 -> top hi code 4 -> 2.0; -3 -> code 0 -> -1.0; 0.4 on lo: (0.4+1)/1.5 = 0.93 -> 1 -> 0.5
    assert Kh[T:, 0].tolist() == [2.0, -1.0, 0.5]


def test_k_channel_grid_error_bound_and_v_untouched():
    r = np.random.default_rng(15)
    T, D, G = 300, 128, 64
    K = (r.standard_normal((T, D)) * r.uniform(0.1, 8, D)).astype(np.float16)
    V = r.standard_normal((T, D)).astype(np.float16).view(np.uint16)
    bm, _, _, _, _ = oracle.select(r.standard_normal(T).astype(np.float32), 0.3)
    kc, _ = oracle.k_channel_grid(K.view(np.uint16), 8, 5)
    hi, lo, _ = oracle.quantize_pack_unit(K.view(np.uint16), V, bm, G, 8, 5, 3, 3, kc=kc)
    hi0, lo0, _ = oracle.quantize_pack_unit(K.view(np.uint16), V, bm, G, 8, 5, 3, 3)
    for a, b in ((hi, hi0), (lo, lo0)):
        assert np.array_equal(a["v"], b["v"]) and np.array_equal(a["vz"], b["vz"])
    Kh, _ = oracle.dequantize_unit(T, D, G, 8, 5, bm, hi, lo, kc=kc)
    is_hi = np.unpackbits(bm.view(np.uint8), bitorder="little")[:T].astype(bool)
    s = np.where(is_hi[:, None], (kc[0] & 0xFFFF).astype(np.uint16).view(np.float16)[None, :],
                 (kc[1] & 0xFFFF).astype(np.uint16).view(np.float16)[None, :]).astype(np.float64)
    err = np.abs(Kh.astype(np.float64) - K.astype(np.float64))
    assert (err <= s / 2 + 1e-6 * (1 + np.abs(K.astype(np.float64)))).all()
