"""GPU parity of the quantizer variants (prior art summarised on the same pages, the SKVQ
abstract): the recent-window selection and the clipped group range, through the C ABI against the
oracle on the same seeded inputs, bit for bit (attention within max-abs 2e-3, rel-L2 1e-3)."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

from gpu_harness import (ATOL, RTOL_L2, attention_errors, check_case, compare_state, fetch, sm_scale,  # noqa: E402
                         to_dev, unit_views)


def _case(B, H, Hq, T, seed, dist="normal"):
    r = np.random.default_rng(seed)
    K = r.standard_normal((B, H, T, 128))
    V = r.standard_normal((B, H, T, 128))
    if dist == "wide":
        K *= 10 ** r.uniform(-3, 3, size=(B, H, T, 1))
        V *= 10 ** r.uniform(-3, 3, size=(B, H, T, 1))
    if dist == "outlier":  # a few large channels, as in real keys
        K[..., r.choice(128, 6, replace=False)] *= 8
    S = r.standard_normal((B, H, T)).astype(np.float32)
    q = r.standard_normal((B, Hq, 128)).astype(np.float16)
    return K.astype(np.float16), V.astype(np.float16), S, q


# ---------------------------------------------------------------- recent window


@pytest.mark.parametrize("B,H,Hq,T,G,L_hi,L_lo,p,W", [
    (1, 2, 8, 700, 64, 8, 5, 0.25, 64),      # one-CTA select
    (2, 1, 4, 3000, 32, 6, 5, 0.1, 300),     # cluster select
    (1, 1, 8, 5000, 128, 16, 8, 0.5, 5000),  # window covers everything
    (1, 2, 16, 2500, 64, 8, 5, 0.0, 129),    # only the window on the finer grid
])
def test_window_full_path(B, H, Hq, T, G, L_hi, L_lo, p, W):
    K, V, S, q = _case(B, H, Hq, T, T + W)
    check_case(K, V, S, q, p, G, L_hi, L_lo, sm_scale(), window=W)


@pytest.mark.parametrize("T", [700, 3000, 20000, 140000])
@pytest.mark.parametrize("p,W", [(0.3, 0), (0.3, 1), (0.3, 517), (0.0, 33), (1.0, 100), (0.5, 10 ** 6)])
def test_window_select_with_ties(T, p, W):
    """Integer scores (many ties, also inside the window) through each select kernel: bitmap,
    rank (and its tail), counts, tau and slot map equal the oracle's."""
    import oracle
    from mixed_precision_kv_semkv_b200 import SemkvCache, semkv_assign_precision

    r = np.random.default_rng(T + W)
    units = 2
    S = r.integers(-4, 4, (1, units, T)).astype(np.float32)
    S[r.random(S.shape) < 0.05] = -0.0
    cache = SemkvCache.for_prefill(1, units, units, 64, 8, 5, T, p, window=W).poison()
    semkv_assign_precision(cache, to_dev(S), T, p)
    bufs = fetch(cache)
    assert cache.status() == 0
    nw, wc = (T + 31) // 32, cache.T_cap // 32
    for u in range(units):
        bm, rk, nh, tau, _ = oracle.select(S[0, u], p, window=W)
        g = unit_views(cache, bufs, u)
        assert np.array_equal(g["bitmap"][:nw], bm) and not g["bitmap"][nw:wc].any(), f"bitmap unit {u}"
        assert np.array_equal(g["rank"][:nw], rk) and (g["rank"][nw:wc] == nh).all(), f"rank unit {u}"
        assert g["n_hi"] == nh and g["n_lo"] == T - nh
        assert np.float32(g["tau"]).view(np.uint32) == np.float32(tau).view(np.uint32)
        bits = np.unpackbits(bm.view(np.uint8), bitorder="little")[:T].astype(bool)
        assert np.array_equal(g["slot_hi"][:nh], np.flatnonzero(bits))
        assert np.array_equal(g["slot_lo"][:T - nh], np.flatnonzero(~bits))


# ---------------------------------------------------------------- clipped range


@pytest.mark.parametrize("B,H,Hq,T,G,L_hi,L_lo,p,clip,dist", [
    (1, 2, 8, 500, 64, 8, 5, 0.25, 0.9, "normal"),
    (2, 1, 4, 333, 32, 6, 5, 0.5, 0.5, "outlier"),
    (1, 1, 8, 640, 128, 16, 8, 0.1, 0.2, "wide"),
    (1, 2, 8, 300, 8, 9, 7, 0.3, 0.75, "normal"),
    (1, 1, 4, 200, 16, 2, 2, 0.5, 0.6, "normal"),
])
def test_clip_full_path(B, H, Hq, T, G, L_hi, L_lo, p, clip, dist):
    K, V, S, q = _case(B, H, Hq, T, int(clip * 1000) + T, dist)
    check_case(K, V, S, q, p, G, L_hi, L_lo, sm_scale(), clip=clip)


def test_clip_one_is_the_plain_path():
    """clip = 1 (and 0) give the plain method's buffers byte for byte."""
    from gpu_harness import run_gpu

    K, V, S, q = _case(1, 2, 8, 400, 3)
    a = run_gpu(K, V, S, q, 0.25, 64, 8, 5, sm_scale())
    b = run_gpu(K, V, S, q, 0.25, 64, 8, 5, sm_scale(), clip=1.0)
    for n in a["bufs"]:
        assert np.array_equal(a["bufs"][n], b["bufs"][n]), n
    assert np.array_equal(a["out"].view(np.uint32), b["out"].view(np.uint32))


@pytest.mark.parametrize("mode", ["append", "append_decode", "running"])
def test_clip_and_window_appends_in_lockstep(mode):
    """Prefill with both variants, then appends (fixed threshold, in one pass with the decode, or
    running top-p) with the clipped grid: state after every step against the oracle's."""
    import torch

    import oracle
    from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_append_decode, semkv_append_token,
                                               semkv_append_token_running, semkv_assign_precision,
                                               semkv_decode_attention, semkv_quantize_pack)

    B, H, Hq, T0, steps, G, L_hi, L_lo, p, W, clip = 1, 2, 8, 260, 90, 64, 8, 5, 0.25, 40, 0.7
    r = np.random.default_rng(77)
    K = r.standard_normal((B, H, T0 + steps, 128)).astype(np.float16)
    V = r.standard_normal((B, H, T0 + steps, 128)).astype(np.float16)
    S = r.standard_normal((B, H, T0 + steps)).astype(np.float32)
    Q = r.standard_normal((steps, B, Hq, 128)).astype(np.float16)
    cache = SemkvCache.for_prefill(B, H, Hq, G, L_hi, L_lo, T0, p, extra=steps, window=W, clip=clip).poison()
    semkv_assign_precision(cache, to_dev(S[:, :, :T0].copy()), T0, p)
    semkv_quantize_pack(cache, to_dev(K[:, :, :T0].copy()), to_dev(V[:, :, :T0].copy()), T0)
    ws = cache.workspace()
    states = []
    for u in range(B * H):
        b, h = divmod(u, H)
        bm, rk, nh, tau, _ = oracle.select(S[b, h, :T0], p, window=W)
        hi, lo, _ = oracle.quantize_pack_unit(K[b, h, :T0].view(np.uint16), V[b, h, :T0].view(np.uint16), bm, G,
                                              L_hi, L_lo, cache.cap_hi // 128, cache.cap_lo // 128, clip=clip)
        states.append(oracle.UnitState(cache.T_cap, bm, rk, nh, T0 - nh, tau, hi, lo))
    g = Hq // H
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
    for s in range(steps):
        t = T0 + s
        k, v, sc, q = (to_dev(x) for x in (K[:, :, t].copy(), V[:, :, t].copy(), S[:, :, t].copy(), Q[s]))
        if mode == "append":
            semkv_append_token(cache, k, v, sc)
        elif mode == "append_decode":
            semkv_append_decode(cache, k, v, sc, q, sm_scale(), out, ws)
        else:
            semkv_append_token_running(cache, k, v, sc, p)
        for u in range(B * H):
            b, h = divmod(u, H)
            kk, vv = K[b, h, t].view(np.uint16), V[b, h, t].view(np.uint16)
            if mode == "running":
                oracle.append_unit_running(states[u], kk, vv, S[b, h, t], p, S[b, h, :t], G, L_hi, L_lo, clip)
            else:
                oracle.append_unit(states[u], kk, vv, S[b, h, t], G, L_hi, L_lo, clip)
    if mode != "append_decode":
        semkv_decode_attention(cache, to_dev(Q[-1]), sm_scale(), out, ws)
    bufs = fetch(cache)
    assert cache.status() == 0
    T = T0 + steps
    for u, st in enumerate(states):
        compare_state(unit_views(cache, bufs, u), {"bitmap": st.bitmap, "rank": st.rank, "n_hi": st.n_hi,
                                                   "tau": st.tau, "hi": st.hi, "lo": st.lo},
                      T, L_hi, L_lo, where=f"unit {u}", strict_tail=False)
        b, h = divmod(u, H)
        Kh, Vh = oracle.dequantize_unit(T, 128, G, L_hi, L_lo, st.bitmap, st.hi, st.lo)
        ref = oracle.attention_fp64(Q[-1, b, h * g:(h + 1) * g].view(np.uint16), Kh, Vh, sm_scale())
        ma, rl = attention_errors(out.cpu().numpy()[b, h * g:(h + 1) * g], ref)
        assert ma <= ATOL and rl <= RTOL_L2, (ma, rl)


# ---------------------------------------------------------------- V level counts of their own


@pytest.mark.parametrize("B,H,Hq,T,G,L_hi,L_lo,L_hi_v,L_lo_v,p", [
    (1, 2, 8, 600, 64, 8, 5, 3, 2, 0.25),    # 2-bit-class keys, 1.5-bit-class values (lo on the tensor cores)
    (1, 2, 8, 900, 64, 8, 5, 4, 2, 0.3),     # both segments on the tensor-core decode with their own V radix
    (2, 2, 16, 400, 128, 8, 6, 5, 4, 0.2),   # g = 8, one group
    (2, 1, 4, 333, 32, 16, 8, 5, 4, 0.5),
    (1, 1, 8, 700, 128, 6, 4, 4, 3, 0.1),
    (1, 2, 8, 500, 64, 8, 5, 8, 3, 0.3),     # hi segment equal (tensor-core decode), lo on its own
    (1, 1, 4, 260, 32, 5, 4, 256, 17, 0.4),  # V finer than K
])
def test_v_levels_full_path(B, H, Hq, T, G, L_hi, L_lo, L_hi_v, L_lo_v, p):
    K, V, S, q = _case(B, H, Hq, T, T + L_hi_v * 7 + L_lo_v)
    check_case(K, V, S, q, p, G, L_hi, L_lo, sm_scale(), L_hi_v=L_hi_v, L_lo_v=L_lo_v)


@pytest.mark.parametrize("Lhv,Llv", [(3, 2), (4, 2)])
@pytest.mark.parametrize("mode", ["append", "append_decode", "running"])
def test_v_levels_appends_in_lockstep(mode, Lhv, Llv):
    import torch

    import oracle
    from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_append_decode, semkv_append_token,
                                               semkv_append_token_running, semkv_assign_precision,
                                               semkv_decode_attention, semkv_quantize_pack)

    B, H, Hq, T0, steps, G, L_hi, L_lo, p = 1, 2, 8, 250, 80, 64, 8, 5, 0.3
    r = np.random.default_rng(78)
    K = r.standard_normal((B, H, T0 + steps, 128)).astype(np.float16)
    V = r.standard_normal((B, H, T0 + steps, 128)).astype(np.float16)
    S = r.standard_normal((B, H, T0 + steps)).astype(np.float32)
    Q = r.standard_normal((steps, B, Hq, 128)).astype(np.float16)
    cache = SemkvCache.for_prefill(B, H, Hq, G, L_hi, L_lo, T0, p, extra=steps, L_hi_v=Lhv, L_lo_v=Llv).poison()
    semkv_assign_precision(cache, to_dev(S[:, :, :T0].copy()), T0, p)
    semkv_quantize_pack(cache, to_dev(K[:, :, :T0].copy()), to_dev(V[:, :, :T0].copy()), T0)
    ws = cache.workspace()
    states = []
    for u in range(B * H):
        b, h = divmod(u, H)
        bm, rk, nh, tau, _ = oracle.select(S[b, h, :T0], p)
        hi, lo, _ = oracle.quantize_pack_unit(K[b, h, :T0].view(np.uint16), V[b, h, :T0].view(np.uint16), bm, G,
                                              L_hi, L_lo, cache.cap_hi // 128, cache.cap_lo // 128, L_hi_v=Lhv,
                                              L_lo_v=Llv)
        states.append(oracle.UnitState(cache.T_cap, bm, rk, nh, T0 - nh, tau, hi, lo))
    g = Hq // H
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
    for s in range(steps):
        t = T0 + s
        k, v, sc, q = (to_dev(x) for x in (K[:, :, t].copy(), V[:, :, t].copy(), S[:, :, t].copy(), Q[s]))
        if mode == "append":
            semkv_append_token(cache, k, v, sc)
        elif mode == "append_decode":
            semkv_append_decode(cache, k, v, sc, q, sm_scale(), out, ws)
        else:
            semkv_append_token_running(cache, k, v, sc, p)
        for u in range(B * H):
            b, h = divmod(u, H)
            kk, vv = K[b, h, t].view(np.uint16), V[b, h, t].view(np.uint16)
            if mode == "running":
                oracle.append_unit_running(states[u], kk, vv, S[b, h, t], p, S[b, h, :t], G, L_hi, L_lo, 1.0, Lhv,
                                           Llv)
            else:
                oracle.append_unit(states[u], kk, vv, S[b, h, t], G, L_hi, L_lo, 1.0, Lhv, Llv)
    if mode != "append_decode":
        semkv_decode_attention(cache, to_dev(Q[-1]), sm_scale(), out, ws)
    bufs = fetch(cache)
    assert cache.status() == 0
    T = T0 + steps
    for u, st in enumerate(states):
        compare_state(unit_views(cache, bufs, u), {"bitmap": st.bitmap, "rank": st.rank, "n_hi": st.n_hi,
                                                   "tau": st.tau, "hi": st.hi, "lo": st.lo},
                      T, L_hi, L_lo, where=f"unit {u}", strict_tail=False, L_hi_v=Lhv, L_lo_v=Llv)
        b, h = divmod(u, H)
        Kh, Vh = oracle.dequantize_unit(T, 128, G, L_hi, L_lo, st.bitmap, st.hi, st.lo, Lhv, Llv)
        ref = oracle.attention_fp64(Q[-1, b, h * g:(h + 1) * g].view(np.uint16), Kh, Vh, sm_scale())
        ma, rl = attention_errors(out.cpu().numpy()[b, h * g:(h + 1) * g], ref)
        assert ma <= ATOL and rl <= RTOL_L2, (ma, rl)


# ---------------------------------------------------------------- per-channel K grids


@pytest.mark.parametrize("B,H,Hq,T,G,L_hi,L_lo,p,clip,dist", [
    (1, 2, 8, 600, 64, 8, 5, 0.25, 0.0, "outlier"),   # a few large key channels
    (2, 1, 4, 333, 32, 6, 5, 0.5, 0.7, "normal"),
    (1, 1, 8, 1500, 128, 16, 4, 0.1, 0.0, "wide"),
])
def test_k_per_channel_full_path(B, H, Hq, T, G, L_hi, L_lo, p, clip, dist):
    K, V, S, q = _case(B, H, Hq, T, T + 91, dist)
    check_case(K, V, S, q, p, G, L_hi, L_lo, sm_scale(), clip=clip, k_per_channel=1)


@pytest.mark.parametrize("mode", ["append", "append_decode", "running"])
def test_k_per_channel_appends_in_lockstep(mode):
    import torch

    import oracle
    from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_append_decode, semkv_append_token,
                                               semkv_append_token_running, semkv_assign_precision,
                                               semkv_decode_attention, semkv_quantize_pack)

    B, H, Hq, T0, steps, G, L_hi, L_lo, p = 1, 2, 8, 260, 70, 64, 8, 5, 0.3
    r = np.random.default_rng(79)
    K = (r.standard_normal((B, H, T0 + steps, 128)) * 1.3).astype(np.float16)  # appends reach past the grid
    V = r.standard_normal((B, H, T0 + steps, 128)).astype(np.float16)
    S = r.standard_normal((B, H, T0 + steps)).astype(np.float32)
    Q = r.standard_normal((steps, B, Hq, 128)).astype(np.float16)
    cache = SemkvCache.for_prefill(B, H, Hq, G, L_hi, L_lo, T0, p, extra=steps, k_per_channel=1).poison()
    semkv_assign_precision(cache, to_dev(S[:, :, :T0].copy()), T0, p)
    semkv_quantize_pack(cache, to_dev(K[:, :, :T0].copy()), to_dev(V[:, :, :T0].copy()), T0)
    ws = cache.workspace()
    states = []
    for u in range(B * H):
        b, h = divmod(u, H)
        bm, rk, nh, tau, _ = oracle.select(S[b, h, :T0], p)
        kc, _ = oracle.k_channel_grid(K[b, h, :T0].view(np.uint16), L_hi, L_lo)
        hi, lo, _ = oracle.quantize_pack_unit(K[b, h, :T0].view(np.uint16), V[b, h, :T0].view(np.uint16), bm, G,
                                              L_hi, L_lo, cache.cap_hi // 128, cache.cap_lo // 128, kc=kc)
        states.append(oracle.UnitState(cache.T_cap, bm, rk, nh, T0 - nh, tau, hi, lo, kc=kc))
    g = Hq // H
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
    for s in range(steps):
        t = T0 + s
        k, v, sc, q = (to_dev(x) for x in (K[:, :, t].copy(), V[:, :, t].copy(), S[:, :, t].copy(), Q[s]))
        if mode == "append":
            semkv_append_token(cache, k, v, sc)
        elif mode == "append_decode":
            semkv_append_decode(cache, k, v, sc, q, sm_scale(), out, ws)
        else:
            semkv_append_token_running(cache, k, v, sc, p)
        for u in range(B * H):
            b, h = divmod(u, H)
            kk, vv = K[b, h, t].view(np.uint16), V[b, h, t].view(np.uint16)
            if mode == "running":
                oracle.append_unit_running(states[u], kk, vv, S[b, h, t], p, S[b, h, :t], G, L_hi, L_lo)
            else:
                oracle.append_unit(states[u], kk, vv, S[b, h, t], G, L_hi, L_lo)
    if mode != "append_decode":
        semkv_decode_attention(cache, to_dev(Q[-1]), sm_scale(), out, ws)
    bufs = fetch(cache)
    assert cache.status() == 0
    T = T0 + steps
    for u, st in enumerate(states):
        compare_state(unit_views(cache, bufs, u), {"bitmap": st.bitmap, "rank": st.rank, "n_hi": st.n_hi,
                                                   "tau": st.tau, "hi": st.hi, "lo": st.lo, "kc": st.kc},
                      T, L_hi, L_lo, where=f"unit {u}", strict_tail=False)
        b, h = divmod(u, H)
        Kh, Vh = oracle.dequantize_unit(T, 128, G, L_hi, L_lo, st.bitmap, st.hi, st.lo, kc=st.kc)
        ref = oracle.attention_fp64(Q[-1, b, h * g:(h + 1) * g].view(np.uint16), Kh, Vh, sm_scale())
        ma, rl = attention_errors(out.cpu().numpy()[b, h * g:(h + 1) * g], ref)
        assert ma <= ATOL and rl <= RTOL_L2, (ma, rl)
