"""Append and attend in one pass (semkv_append_decode): the decode CTA that holds the new token's
slot quantizes and writes the token before it reads that tile; the merge does the unit's
bookkeeping.  Its results must be those of semkv_append_token followed by semkv_decode_attention:
compared bit for bit with the two calls step by step, and with the oracle at the end."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["i8", "tc"])
def decode_path(request, monkeypatch):
    """Every case through both tensor-core decodes: the integer one ("i8") wherever it serves the
    shape, and the fp16 one ("tc"); by default the library picks one by the tile count."""
    monkeypatch.setenv("SEMKV_DECODE", request.param)
    return request.param


def _run(B, H, Hq, T0, steps, G, L_hi, L_lo, p, extra, seed):
    import torch

    from gpu_harness import fetch, sm_scale, to_dev
    from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_append_decode, semkv_append_token,
                                               semkv_assign_precision, semkv_decode_attention, semkv_quantize_pack)

    r = np.random.default_rng(seed)
    K = r.standard_normal((B, H, T0 + steps, 128)).astype(np.float16)
    V = r.standard_normal((B, H, T0 + steps, 128)).astype(np.float16)
    S = r.standard_normal((B, H, T0 + steps)).astype(np.float32)
    Q = r.standard_normal((steps, B, Hq, 128)).astype(np.float16)
    caches = []
    for _ in range(2):
        c = SemkvCache.for_prefill(B, H, Hq, G, L_hi, L_lo, T0, p, extra=extra).poison()
        semkv_assign_precision(c, to_dev(S[:, :, :T0].copy()), T0, p)
        semkv_quantize_pack(c, to_dev(K[:, :, :T0].copy()), to_dev(V[:, :, :T0].copy()), T0)
        caches.append(c)
    fused, split = caches
    ws_f, ws_s = fused.workspace(), split.workspace()
    outs = []
    for s in range(steps):
        t = T0 + s
        k, v, sc, q = (to_dev(x) for x in (K[:, :, t].copy(), V[:, :, t].copy(), S[:, :, t].copy(), Q[s]))
        of = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
        os_ = torch.empty_like(of)
        semkv_append_decode(fused, k, v, sc, q, sm_scale(), of, ws_f)
        semkv_append_token(split, k, v, sc)
        semkv_decode_attention(split, q, sm_scale(), os_, ws_s)
        a, b = of.cpu().numpy(), os_.cpu().numpy()
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), f"step {s}"
        outs.append(a)
    bf, bs = fetch(fused), fetch(split)
    assert fused.status() == split.status()
    for name in bf:
        if name in ("slot_token",):  # not part of the state after appends (prefill only)
            continue
        assert np.array_equal(bf[name], bs[name]), name
    return fused, bf, outs, (K, V, S, Q)


@pytest.mark.parametrize("p,L_hi,L_lo,G", [(0.25, 8, 5, 64), (0.5, 6, 5, 128), (0.1, 16, 4, 32)])
def test_fused_equals_two_calls_and_oracle(p, L_hi, L_lo, G):
    import oracle
    from gpu_harness import attention_errors, compare_state, sm_scale, unit_views

    B, H, Hq, T0, steps = 2, 2, 8, 250, 140
    fused, bufs, outs, (K, V, S, Q) = _run(B, H, Hq, T0, steps, G, L_hi, L_lo, p, extra=160, seed=21)
    assert fused.status() == 0
    g = Hq // H
    T = T0 + steps
    for u in range(B * H):
        b, h = divmod(u, H)
        bm, rk, nh, tau, _ = oracle.select(S[b, h, :T0], p)
        hi, lo, _ = oracle.quantize_pack_unit(K[b, h, :T0].view(np.uint16), V[b, h, :T0].view(np.uint16), bm, G,
                                              L_hi, L_lo, fused.cap_hi // 128, fused.cap_lo // 128)
        st = oracle.UnitState(fused.T_cap, bm, rk, nh, T0 - nh, tau, hi, lo)
        for s in range(steps):
            t = T0 + s
            oracle.append_unit(st, K[b, h, t].view(np.uint16), V[b, h, t].view(np.uint16), S[b, h, t], G, L_hi, L_lo)
            if s in (0, steps // 2, steps - 1):
                Kh, Vh = oracle.dequantize_unit(t + 1, 128, G, L_hi, L_lo, st.bitmap, st.hi, st.lo)
                ref = oracle.attention_fp64(Q[s, b, h * g:(h + 1) * g].view(np.uint16), Kh, Vh, sm_scale())
                ma, rl = attention_errors(outs[s][b, h * g:(h + 1) * g], ref)
                assert ma <= 2e-3 and rl <= 1e-3, (s, ma, rl)
        compare_state(unit_views(fused, bufs, u), {"bitmap": st.bitmap, "rank": st.rank, "n_hi": st.n_hi,
                                                   "tau": st.tau, "hi": st.hi, "lo": st.lo},
                      T, L_hi, L_lo, where=f"unit {u}", strict_tail=False)


def test_fused_overflow_matches_two_calls():
    # p = 0: every token goes lo; the lo segment (128 slots) fills after 8 appends
    fused, _, _, _ = _run(1, 1, 4, 120, 20, 64, 8, 5, 0.0, extra=0, seed=5)
    assert fused.status() & 4


def test_fused_falls_back_on_other_shapes():
    # L = 9 has no tensor-core decode: the call runs append then decode
    _run(1, 2, 8, 300, 12, 64, 9, 7, 0.25, extra=64, seed=6)
