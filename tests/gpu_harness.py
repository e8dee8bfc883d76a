"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and the oracle on
the same inputs, and compare (bit-exact for bitmaps, ranks, counts, thresholds, packed words,
scale/zero and dequantized values; attention within max-abs 2e-3 and relative L2 1e-3 of fp64)."""
from __future__ import annotations

import math

import numpy as np

import oracle
from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_append_token, semkv_assign_precision,
                                           semkv_decode_attention, semkv_dequantize, semkv_quantize_pack)

ATOL = 2e-3
RTOL_L2 = 1e-3


def to_dev(a):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def unit_views(cache: SemkvCache, bufs: dict, u: int):
    """Per-unit numpy views of the fetched device buffers, in the oracle's array shapes."""
    B, H, G, D = cache.B, cache.H, cache.G, cache.D
    units = B * H
    out = {}
    for seg, L, Lv, cap in (("hi", cache.L_hi, cache.L_hi_v, cache.cap_hi), ("lo", cache.L_lo, cache.L_lo_v,
                                                                             cache.cap_lo)):
        tiles = cap // 128
        sh = oracle.segment_shapes(D, G, L, tiles, Lv)
        d = {}
        for name in ("k", "v", "kz", "vz"):
            arr = bufs[f"{name}_{seg}"].view(np.uint32)
            per = int(np.prod(sh[name]))
            d[name] = arr[: units * per].reshape(units, *sh[name])[u]
        out[seg] = d
    wc = cache.T_cap // 32
    out["bitmap"] = bufs["bitmap"].view(np.uint32)[: units * wc].reshape(units, wc)[u]
    out["rank"] = bufs["rank"].view(np.uint32)[: units * wc].reshape(units, wc)[u]
    out["n_hi"] = int(bufs["n_hi"][u])
    out["n_lo"] = int(bufs["n_lo"][u])
    out["tau"] = np.float32(bufs["tau"].view(np.float32)[u])
    caps = cache.cap_hi + cache.cap_lo
    st = bufs["slot_token"].view(np.int32)[: units * caps].reshape(units, caps)[u]
    out["slot_hi"], out["slot_lo"] = st[: cache.cap_hi], st[cache.cap_hi:]
    out["kc"] = bufs["kc"].view(np.uint32)[: units * 2 * D].reshape(units, 2, D)[u]
    return out


def fetch(cache: SemkvCache) -> dict:
    import torch

    torch.cuda.synchronize()
    return {n: t.cpu().numpy() for n, t in cache.bufs.items()}


def run_gpu(K, V, S, q, p, G, L_hi, L_lo, scale, extra=0, window=0, clip=0.0, L_hi_v=0, L_lo_v=0, k_per_channel=0):
    import torch

    B, H, T, D = K.shape
    Hq = q.shape[1]
    cache = SemkvCache.for_prefill(B, H, Hq, G, L_hi, L_lo, T, p, extra=extra, window=window, clip=clip,
                                   L_hi_v=L_hi_v, L_lo_v=L_lo_v, k_per_channel=k_per_channel).poison()
    dK, dV, dS, dq = to_dev(K), to_dev(V), to_dev(S), to_dev(q)
    semkv_assign_precision(cache, dS, T, p)
    semkv_quantize_pack(cache, dK, dV, T)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
    ws = cache.workspace()
    semkv_decode_attention(cache, dq, scale, out, ws)
    Kh = torch.empty((B, H, T, D), dtype=torch.float32, device="cuda")
    Vh = torch.empty_like(Kh)
    semkv_dequantize(cache, Kh, Vh, T)
    res = {"cache": cache, "bufs": fetch(cache), "out": out.cpu().numpy(), "Kh": Kh.cpu().numpy(),
           "Vh": Vh.cpu().numpy(), "status": cache.status()}
    return res


def oracle_unit(K, V, S, q, p, G, L_hi, L_lo, scale, tiles_hi, tiles_lo, window=0, clip=0.0, L_hi_v=0, L_lo_v=0,
                k_per_channel=0):
    """Oracle results of one unit. K, V [T][D] fp16; S [T]; q [g][D] fp16.  window, clip, L_hi_v,
    L_lo_v, k_per_channel: the quantizer variants as the cache fields state them (0 = off)."""
    bm, rk, nh, tau, st = oracle.select(S, p, window=window)
    kc = oracle.k_channel_grid(K.view(np.uint16), L_hi, L_lo, clip or 1.0)[0] if k_per_channel else None
    hi, lo, st2 = oracle.quantize_pack_unit(K.view(np.uint16), V.view(np.uint16), bm, G, L_hi, L_lo, tiles_hi,
                                            tiles_lo, clip=clip or 1.0, L_hi_v=L_hi_v or None, L_lo_v=L_lo_v or None,
                                            kc=kc)
    T = K.shape[0]
    Kh, Vh = oracle.dequantize_unit(T, K.shape[1], G, L_hi, L_lo, bm, hi, lo, L_hi_v or None, L_lo_v or None, kc=kc)
    o = oracle.attention_fp64(q.view(np.uint16), Kh, Vh, scale)
    res = {"bitmap": bm, "rank": rk, "n_hi": nh, "tau": tau, "hi": hi, "lo": lo, "Kh": Kh, "Vh": Vh, "out": o,
           "status": st | st2}
    if kc is not None:
        res["kc"] = kc
    return res


def _words_equal(a, b, what):
    if not np.array_equal(a, b):
        bad = np.argwhere(a != b)
        raise AssertionError(f"{what}: {len(bad)} words differ, first at {bad[0].tolist()} "
                             f"gpu={a[tuple(bad[0])]:#x} oracle={b[tuple(bad[0])]:#x}")


def compare_state(g: dict, o: dict, T: int, L_hi: int, L_lo: int, where: str = "", strict_tail: bool = True,
                  L_hi_v: int = 0, L_lo_v: int = 0):
    """Bit-exact comparison of one unit's state.  strict_tail: the last tile's slots past n must be
    zero as well (true after a prefill; after appends into a new tile they are unspecified, except
    that V words holding a live slot have zero digits past n)."""
    nw = (T + 31) // 32
    assert np.array_equal(g["bitmap"][:nw], o["bitmap"][:nw]), f"bitmap {where}"
    assert np.array_equal(g["rank"][:nw], o["rank"][:nw]), f"rank {where}"
    assert g["n_hi"] == o["n_hi"] and g["n_lo"] == T - o["n_hi"], f"counts {where}"
    assert np.float32(g["tau"]).view(np.uint32) == np.float32(o["tau"]).view(np.uint32), f"tau {where}"
    if o.get("kc") is not None:
        _words_equal(g["kc"], o["kc"], f"per-channel K grids {where}")
    if strict_tail and "slot_hi" in g:  # after a prefill: the slot map is the inverse of the ranks
        bits = np.unpackbits(o["bitmap"][:nw].view(np.uint8), bitorder="little")[:T].astype(bool)
        tokens = np.arange(T)
        assert np.array_equal(g["slot_hi"][: o["n_hi"]], tokens[bits]), f"slot map hi {where}"
        assert np.array_equal(g["slot_lo"][: T - o["n_hi"]], tokens[~bits]), f"slot map lo {where}"
    for seg, n, L in (("hi", o["n_hi"], L_hi_v or L_hi), ("lo", T - o["n_hi"], L_lo_v or L_lo)):  # L: V's
        if strict_tail:
            nt = -(-n // 128)
            for name in ("k", "v", "kz", "vz"):
                _words_equal(g[seg][name][:nt], o[seg][name][:nt], f"{seg}.{name} {where}")
            continue
        full, rem = divmod(n, 128)
        k = oracle.radix_digits(L)
        for name in ("k", "v", "kz", "vz"):
            _words_equal(g[seg][name][:full], o[seg][name][:full], f"{seg}.{name} {where}")
        if rem:
            for name in ("k", "kz", "vz"):
                _words_equal(g[seg][name][full][:, :rem], o[seg][name][full][:, :rem], f"{seg}.{name} tail {where}")
            nwv = -(-rem // k)
            _words_equal(g[seg]["v"][full][:nwv], o[seg]["v"][full][:nwv], f"{seg}.v tail {where}")


def attention_errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    max_abs = float(np.abs(got - ref).max()) if got.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got - ref))
    return max_abs, rel


def check_case(K, V, S, q, p, G, L_hi, L_lo, scale, units=None, window=0, clip=0.0, L_hi_v=0, L_lo_v=0,
               k_per_channel=0):
    """Run the GPU path on a whole case and compare the chosen units (default: all) with the oracle."""
    B, H, T, D = K.shape
    g = q.shape[1] // H
    res = run_gpu(K, V, S, q, p, G, L_hi, L_lo, scale, window=window, clip=clip, L_hi_v=L_hi_v, L_lo_v=L_lo_v,
                  k_per_channel=k_per_channel)
    cache = res["cache"]
    assert res["status"] == 0, f"status {res['status']}"
    units = range(B * H) if units is None else units
    worst = (0.0, 0.0)
    for u in units:
        b, h = divmod(u, H)
        o = oracle_unit(K[b, h], V[b, h], S[b, h], q[b, h * g:(h + 1) * g], p, G, L_hi, L_lo, scale,
                        cache.cap_hi // 128, cache.cap_lo // 128, window=window, clip=clip, L_hi_v=L_hi_v,
                        L_lo_v=L_lo_v, k_per_channel=k_per_channel)
        gu = unit_views(cache, res["bufs"], u)
        compare_state(gu, o, T, L_hi, L_lo, where=f"unit {u}", L_hi_v=L_hi_v, L_lo_v=L_lo_v)
        assert np.array_equal(res["Kh"][b, h].view(np.uint32), o["Kh"].view(np.uint32)), f"Khat unit {u}"
        assert np.array_equal(res["Vh"][b, h].view(np.uint32), o["Vh"].view(np.uint32)), f"Vhat unit {u}"
        ma, rl = attention_errors(res["out"][b, h * g:(h + 1) * g], o["out"])
        worst = (max(worst[0], ma), max(worst[1], rl))
        assert ma <= ATOL and rl <= RTOL_L2, f"attention unit {u}: max_abs {ma:.3g} rel_l2 {rl:.3g}"
    return worst


def sm_scale(D=128):
    return 1.0 / math.sqrt(D)
