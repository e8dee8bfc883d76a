"""Running top-p for generated tokens (the exact reading of a running threshold): the new token goes
on the finer grid iff it is among the floor(p (T+1)) largest of all T+1 scores, ties to the lower
token index (so the new token loses them); earlier tokens keep their grid.

CPU pins of the oracle (brute force over explicit orderings, the count identity the kernel uses,
the p = 0 and p = 1 ends) and the GPU path in lockstep with the oracle."""
import math

import numpy as np
import pytest


def _brute(prev, new, p):
    T = len(prev)
    order = sorted(range(T + 1), key=lambda i: (-(float(prev[i]) if i < T else float(new)), i))
    return T in order[: math.floor(p * (T + 1))]


def test_oracle_matches_brute_force_on_small_cases(orc):
    r = np.random.default_rng(3)
    for trial in range(400):
        T = int(r.integers(0, 13))
        vals = r.integers(0, 4, size=T + 1).astype(np.float32) - 1.5  # few values: many ties
        if trial % 3 == 0:
            vals = r.standard_normal(T + 1).astype(np.float32)
        if trial % 7 == 0 and T > 0:
            vals[-1] = -0.0
            vals[0] = 0.0
        p = float(r.choice([0.0, 0.1, 0.25, 0.5, 0.75, 0.9, 1.0, r.random()]))
        assert orc.running_is_hi(vals[:T], float(vals[T]), p) == _brute(vals[:T], vals[T], p), (vals, p)


def test_count_identity_used_by_the_kernel(orc):
    """new is hi  iff  #{earlier scores >= new} < floor(p (T+1))  (-0 == +0)."""
    r = np.random.default_rng(4)
    for _ in range(300):
        T = int(r.integers(1, 200))
        vals = (r.integers(0, 9, size=T + 1) - 4).astype(np.float32) * np.float32(0.5)
        p = float(r.random())
        cnt = int(np.sum(vals[:T] >= vals[T]))
        assert orc.running_is_hi(vals[:T], float(vals[T]), p) == (cnt < math.floor(p * (T + 1)))


def test_ends(orc):
    r = np.random.default_rng(5)
    prev = r.standard_normal(50).astype(np.float32)
    for new in (-10.0, 0.0, 10.0):
        assert not orc.running_is_hi(prev, new, 0.0)
        assert orc.running_is_hi(prev, new, 1.0)


@pytest.mark.gpu
@pytest.mark.parametrize("p,L_hi,L_lo,G", [(0.25, 8, 5, 64), (0.5, 6, 5, 128), (0.1, 16, 3, 32)])
def test_running_appends_match_oracle_in_lockstep(p, L_hi, L_lo, G):
    import torch

    import oracle
    from gpu_harness import attention_errors, compare_state, fetch, sm_scale, to_dev, unit_views
    from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_append_token_running, semkv_assign_precision,
                                               semkv_decode_attention, semkv_quantize_pack)

    B, H, Hq, T0, steps = 2, 2, 8, 300, 200
    r = np.random.default_rng(11)
    K = r.standard_normal((B, H, T0 + steps, 128)).astype(np.float16)
    V = r.standard_normal((B, H, T0 + steps, 128)).astype(np.float16)
    S = r.standard_normal((B, H, T0 + steps)).astype(np.float32)
    S[:, :, T0 + 5] = S[:, :, 17]  # a tie with an earlier token: the new one loses it
    q = r.standard_normal((B, Hq, 128)).astype(np.float16)
    g = Hq // H
    cache = SemkvCache.for_prefill(B, H, Hq, G, L_hi, L_lo, T0, p, extra=steps + 64).poison()
    semkv_assign_precision(cache, to_dev(S[:, :, :T0].copy()), T0, p)
    semkv_quantize_pack(cache, to_dev(K[:, :, :T0].copy()), to_dev(V[:, :, :T0].copy()), T0)
    for t in range(T0, T0 + steps):
        semkv_append_token_running(cache, to_dev(K[:, :, t].copy()), to_dev(V[:, :, t].copy()),
                                   to_dev(S[:, :, t].copy()), p)
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
    semkv_decode_attention(cache, to_dev(q), sm_scale(), out, cache.workspace())
    bufs = fetch(cache)
    assert cache.status() == 0
    T = T0 + steps
    keys = bufs["score_keys"].view(np.uint32).reshape(B * H, cache.T_cap)
    for u in range(B * H):
        b, h = divmod(u, H)
        bm, rk, nh, tau, _ = oracle.select(S[b, h, :T0], p)
        hi, lo, _ = oracle.quantize_pack_unit(K[b, h, :T0].view(np.uint16), V[b, h, :T0].view(np.uint16), bm, G,
                                              L_hi, L_lo, cache.cap_hi // 128, cache.cap_lo // 128)
        st = oracle.UnitState(cache.T_cap, bm, rk, nh, T0 - nh, tau, hi, lo)
        for t in range(T0, T):
            oracle.append_unit_running(st, K[b, h, t].view(np.uint16), V[b, h, t].view(np.uint16), float(S[b, h, t]),
                                       p, S[b, h, :t], G, L_hi, L_lo)
        gu = unit_views(cache, bufs, u)
        assert gu["n_hi"] == st.n_hi and gu["n_lo"] == st.n_lo
        compare_state(gu, {"bitmap": st.bitmap, "rank": st.rank, "n_hi": st.n_hi, "tau": st.tau, "hi": st.hi,
                           "lo": st.lo}, T, L_hi, L_lo, where=f"unit {u}", strict_tail=False)
        # the stored keys order exactly as the scores (-0 as +0)
        kv = keys[u, :T].astype(np.int64)
        sv = S[b, h, :T].astype(np.float64)
        i, j = r.integers(0, T, size=(2, 4000))
        assert np.all((kv[i] > kv[j]) == (sv[i] > sv[j])) and np.all((kv[i] == kv[j]) == (sv[i] == sv[j]))
        Kh, Vh = oracle.dequantize_unit(T, 128, G, L_hi, L_lo, st.bitmap, st.hi, st.lo)
        ref = oracle.attention_fp64(q[b, h * g:(h + 1) * g].view(np.uint16), Kh, Vh, sm_scale())
        ma, rl = attention_errors(out.cpu().numpy()[b, h * g:(h + 1) * g], ref)
        assert ma <= 2e-3 and rl <= 1e-3, (ma, rl)
