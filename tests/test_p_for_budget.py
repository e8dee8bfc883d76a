"""Storage-budget helper: the largest fraction p on the finer grid whose storage reduction against
fp16 still meets a target (SemKV page, Abstract: measure the cliff, then interpolate above it).

The oracle finds p by bisection on the storage it counts from its own buffer shapes; the library
inverts the closed form.  Pins: the round trip through the oracle's storage, the p = 0 and p = 1
ends, monotonicity in the target, and the buffer bytes of a prefill made with the returned p."""
import math

import numpy as np
import pytest

PAIRS = [(6, 5), (8, 6), (16, 8), (8, 5), (5, 4), (5, 5), (4, 8)]


@pytest.mark.parametrize("L_hi,L_lo", PAIRS)
@pytest.mark.parametrize("G", [32, 64, 128])
def test_library_matches_oracle_bisection(semkv, orc, L_hi, L_lo, G):
    lo_r = 16.0 / orc.storage_bits_per_value(128, G, L_hi, L_lo, 1.0)
    hi_r = 16.0 / orc.storage_bits_per_value(128, G, L_hi, L_lo, 0.0)
    a, b = min(lo_r, hi_r), max(lo_r, hi_r)
    for ratio in np.linspace(a * 0.9, b * 1.001, 23):
        want = orc.p_for_ratio(128, G, L_hi, L_lo, float(ratio))
        if want is None:
            with pytest.raises(semkv.SemkvError) as e:
                semkv.semkv_p_for_ratio(128, G, L_hi, L_lo, float(ratio))
            assert e.value.code == semkv._lib.SEMKV_ERR_CAPACITY
            continue
        got = semkv.semkv_p_for_ratio(128, G, L_hi, L_lo, float(ratio))
        assert 0.0 <= got <= 1.0
        assert abs(got - want) < 1e-9, (ratio, got, want)


@pytest.mark.parametrize("L_hi,L_lo,G", [(6, 5, 64), (8, 6, 32), (16, 8, 128)])
def test_round_trip_and_ends(orc, L_hi, L_lo, G):
    for p in (0.0, 0.1, 0.25, 0.5, 0.75, 0.9, 1.0):
        ratio = 16.0 / orc.storage_bits_per_value(128, G, L_hi, L_lo, p)
        got = orc.p_for_ratio(128, G, L_hi, L_lo, ratio)
        assert abs(got - p) < 1e-9
    # a target above the coarse grid's own reduction is out of reach
    r0 = 16.0 / orc.storage_bits_per_value(128, G, L_hi, L_lo, 0.0)
    assert orc.p_for_ratio(128, G, L_hi, L_lo, r0 * 1.0001) is None
    # a target at or below the fine grid's reduction leaves every token on the fine grid
    r1 = 16.0 / orc.storage_bits_per_value(128, G, L_hi, L_lo, 1.0)
    assert orc.p_for_ratio(128, G, L_hi, L_lo, r1) == 1.0
    assert orc.p_for_ratio(128, G, L_hi, L_lo, r1 * 0.5) == 1.0


def test_more_compression_leaves_less_for_the_fine_grid(orc):
    prev = 1.0
    for ratio in np.linspace(4.3, 5.3, 21):
        p = orc.p_for_ratio(128, 64, 6, 5, float(ratio))
        assert p is not None and p <= prev + 1e-15
        prev = p


def test_prefill_at_the_returned_p_meets_the_budget(semkv, orc):
    """Buffer bytes of a prefill made with floor(p*T) fine tokens give at least the target ratio."""
    T, G, L_hi, L_lo = 128 * 64, 64, 8, 5
    for ratio in (4.5, 4.8, 5.0, 5.2):
        p = semkv.semkv_p_for_ratio(128, G, L_hi, L_lo, ratio)
        nh = orc.n_hi(p, T)
        hi = orc.segment_shapes(128, G, L_hi, math.ceil(nh / 128))
        lo = orc.segment_shapes(128, G, L_lo, math.ceil((T - nh) / 128))
        # bytes of the tokens actually stored (full tiles plus the used part of the last ones)
        per_tok = lambda sh: sum(int(np.prod(s)) for s in sh.values()) * 32 / max(1, sh["k"][0] * 128)  # noqa: E731
        bits = (nh * per_tok(hi) + (T - nh) * per_tok(lo) + T) / (2 * T * 128)
        assert 16.0 / bits >= ratio - 1e-9, (ratio, p, 16.0 / bits)


def test_bad_arguments(semkv):
    E = semkv.SemkvError
    for args in ((128, 64, 8, 5, 0.0), (128, 64, 8, 5, -1.0), (128, 64, 8, 5, float("nan")), (128, 48, 8, 5, 5.0),
                 (0, 64, 8, 5, 5.0)):
        with pytest.raises(E) as e:
            semkv.semkv_p_for_ratio(*args)
        assert e.value.code == semkv._lib.SEMKV_ERR_INVALID_ARG
    with pytest.raises(E) as e:
        semkv.semkv_p_for_ratio(128, 64, 257, 5, 5.0)
    assert e.value.code == semkv._lib.SEMKV_ERR_UNSUPPORTED


@pytest.mark.parametrize("L_hi,L_lo,L_hi_v,L_lo_v", [(8, 5, 3, 2), (6, 5, 6, 3), (16, 8, 5, 4), (5, 4, 8, 6)])
def test_library_matches_oracle_bisection_with_v_levels(semkv, orc, L_hi, L_lo, L_hi_v, L_lo_v):
    G = 64
    r1 = 16.0 / orc.storage_bits_per_value(128, G, L_hi, L_lo, 1.0, L_hi_v, L_lo_v)
    r0 = 16.0 / orc.storage_bits_per_value(128, G, L_hi, L_lo, 0.0, L_hi_v, L_lo_v)
    a, b = min(r0, r1), max(r0, r1)
    for ratio in np.linspace(a * 0.9, b * 1.001, 19):
        want = orc.p_for_ratio(128, G, L_hi, L_lo, float(ratio), L_hi_v=L_hi_v, L_lo_v=L_lo_v)
        if want is None:
            with pytest.raises(semkv.SemkvError):
                semkv.semkv_p_for_ratio_kv(128, G, L_hi, L_lo, L_hi_v, L_lo_v, float(ratio))
            continue
        got = semkv.semkv_p_for_ratio_kv(128, G, L_hi, L_lo, L_hi_v, L_lo_v, float(ratio))
        assert abs(got - want) < 1e-9, (ratio, got, want)
    # equal counts: the plain helper
    assert semkv.semkv_p_for_ratio_kv(128, G, 8, 5, 8, 5, 4.8) == semkv.semkv_p_for_ratio(128, G, 8, 5, 4.8)
