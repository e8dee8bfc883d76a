"""GPU parity: every output of the CUDA path, called through the C ABI, against the CPU oracle on
the same seeded inputs.  Bit-exact for bitmaps, ranks, counts, thresholds, packed words,
scale/zero and dequantized values; decode attention within max-abs 2e-3 and relative L2 1e-3 of
the oracle's fp64 attention over the same dequantized K/V."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

from gpu_harness import (ATOL, RTOL_L2, attention_errors, check_case, compare_state, fetch, oracle_unit,  # noqa: E402
                         run_gpu, sm_scale, to_dev, unit_views)


def _rand_case(B, H, Hq, T, seed, dist="normal"):
    r = np.random.default_rng(seed)
    K = r.standard_normal((B, H, T, 128))
    V = r.standard_normal((B, H, T, 128))
    if dist == "wide":
        K *= 10 ** r.uniform(-3, 3, size=(B, H, T, 1))
        V *= 10 ** r.uniform(-3, 3, size=(B, H, T, 1))
    S = r.standard_normal((B, H, T)).astype(np.float32)
    q = r.standard_normal((B, Hq, 128)).astype(np.float16)
    return K.astype(np.float16), V.astype(np.float16), S, q


@pytest.fixture(autouse=True, params=["i8", "tc"])
def decode_path(request, monkeypatch):
    """Every case through both tensor-core decodes: the integer one ("i8") wherever it serves the
    shape, and the fp16 one ("tc"); by default the library picks one by the tile count."""
    monkeypatch.setenv("SEMKV_DECODE", request.param)
    return request.param


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch

    from mixed_precision_kv_semkv_b200 import build

    build.build()
    assert torch.cuda.is_available()


def test_tiny_workload_all_outputs():
    from mixed_precision_kv_semkv_b200 import synth

    w = synth.WORKLOADS["tiny"]
    d = synth.layer_cpu(w, 0)
    check_case(d["K"], d["V"], d["scores"], d["q"], w.p, w.G, w.L_hi, w.L_lo, synth.sm_scale())


@pytest.mark.parametrize("B,H,Hq,T,G,L_hi,L_lo,p", [
    (1, 2, 8, 1, 128, 8, 5, 0.5),
    (1, 1, 4, 31, 64, 8, 5, 0.5),
    (2, 2, 4, 33, 32, 6, 5, 0.25),
    (1, 2, 2, 300, 16, 16, 8, 0.75),
    (1, 1, 1, 1000, 8, 4, 3, 0.3),
    (1, 1, 8, 2000, 128, 9, 7, 0.1),
    (1, 2, 8, 777, 64, 8, 5, 0.0),
    (1, 2, 8, 777, 64, 8, 5, 1.0),
    (1, 1, 4, 700, 64, 256, 17, 0.5),
    (1, 1, 4, 500, 32, 100, 31, 0.4),
    (3, 1, 2, 4095, 64, 8, 5, 0.25),
    (1, 1, 4, 20000, 64, 8, 5, 0.25),     # selection: keys cached in shared memory
    (1, 1, 4, 140000, 128, 6, 5, 0.5),    # selection: scores streamed (more than a cluster holds)
])
def test_ragged_shapes_and_levels(B, H, Hq, T, G, L_hi, L_lo, p):
    K, V, S, q = _rand_case(B, H, Hq, T, seed=T + L_hi)
    check_case(K, V, S, q, p, G, L_hi, L_lo, sm_scale())


@pytest.mark.parametrize("L", list(range(3, 17)))
def test_every_small_level_pair(L):
    K, V, S, q = _rand_case(1, 1, 4, 600, seed=L, dist="wide")
    check_case(K, V, S, q, 0.5, 32, L, L - 1, sm_scale())


@pytest.mark.parametrize("kind", ["all_equal", "few_values", "signed_zeros"])
def test_score_ties(kind):
    K, V, S, q = _rand_case(1, 2, 8, 1500, seed=7)
    r = np.random.default_rng(1)
    if kind == "all_equal":
        S[:] = 0.5
    elif kind == "few_values":
        S = np.array([0.0, 1.0, 2.0], np.float32)[r.integers(0, 3, size=S.shape)]
    else:
        S = np.array([-0.0, 0.0, 1.0], np.float32)[r.integers(0, 3, size=S.shape)]
    check_case(K, V, S, q, 0.4, 64, 8, 5, sm_scale())


def test_constant_and_extreme_groups():
    K, V, S, q = _rand_case(1, 1, 4, 256, seed=3)
    K[0, 0, :10] = 1.5          # constant rows: zero scale
    V[0, 0, 10:20] = -0.0
    K[0, 0, 20, :64] = 65504.0  # huge range: scale saturates
    K[0, 0, 20, 64:] = -65504.0
    V[0, 0, 21] = np.float16(6e-8)  # subnormal values
    check_case(K, V, S, q, 0.5, 64, 8, 5, sm_scale())


@pytest.mark.parametrize("L", [3, 4, 5, 6, 8, 16])
def test_quotients_at_and_near_half_steps(L):
    """Values at, and one fp16 step around, the half-way points between grid levels: the codes
    depend on the exact IEEE quotient and on ties-to-even, so any other division rule shows up."""
    import oracle

    r = np.random.default_rng(100 + L)
    T, G = 384, 64
    K = np.empty((1, 1, T, 128), np.float16)
    for t in range(T):
        for grp in range(2):
            mn = np.float16(r.standard_normal() * 2)
            mx = np.float16(float(mn) + abs(r.standard_normal()) * 4 + 0.01)
            probe = np.array([mn, mx] * (G // 2), np.float16)
            _, s16, _, _ = oracle.quantize_group(probe.view(np.uint16), L)
            s = float(np.uint16(s16).view(np.float16))
            c = r.integers(0, L - 1, size=G)
            x = (float(mn) + (c + 0.5) * s).astype(np.float16)
            nudge = r.integers(-1, 2, size=G)  # -1, 0, +1 fp16 step
            x = np.where(nudge < 0, np.nextafter(x, np.float16(-np.inf)),
                         np.where(nudge > 0, np.nextafter(x, np.float16(np.inf)), x))
            x = np.clip(x, mn, mx)
            x[0], x[1] = mn, mx
            K[0, 0, t, grp * G:(grp + 1) * G] = x
    V = K[:, :, ::-1].copy()
    S = r.standard_normal((1, 1, T)).astype(np.float32)
    q = r.standard_normal((1, 4, 128)).astype(np.float16)
    check_case(K, V, S, q, 0.5, G, L, max(2, L - 1), sm_scale())


def test_device_status_flags():
    import torch

    K, V, S, q = _rand_case(1, 1, 4, 64, seed=5)
    S[0, 0, 3] = np.nan
    V[0, 0, 9, 7] = np.inf
    res = run_gpu(K, V, S, q, 0.5, 64, 8, 5, sm_scale())
    assert res["status"] & 1 and res["status"] & 2
    torch.cuda.synchronize()


def test_llama8b_layer_full_size():
    """The bench workload (one Llama-3.1-8B-shaped layer, T=32768, G64, L 8/5, p 0.25): all units."""
    from mixed_precision_kv_semkv_b200 import synth

    w = synth.WORKLOADS["llama8b_1L"]
    d = synth.layer_cpu(w, 0)
    worst = check_case(d["K"], d["V"], d["scores"], d["q"], w.p, w.G, w.L_hi, w.L_lo, synth.sm_scale())
    assert worst[0] <= ATOL and worst[1] <= RTOL_L2


# ---------------------------------------------------------------- append (generation-time quantization)


def _append_lockstep(B, H, Hq, T0, steps, G, L_hi, L_lo, p, seed, extra):
    import torch

    import oracle
    from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_append_token, semkv_assign_precision,
                                               semkv_decode_attention, semkv_quantize_pack)

    r = np.random.default_rng(seed)
    K = r.standard_normal((B, H, T0 + steps, 128)).astype(np.float16)
    V = r.standard_normal((B, H, T0 + steps, 128)).astype(np.float16)
    S = r.standard_normal((B, H, T0 + steps)).astype(np.float32)
    q = r.standard_normal((B, Hq, 128)).astype(np.float16)
    g = Hq // H
    cache = SemkvCache.for_prefill(B, H, Hq, G, L_hi, L_lo, T0, p, extra=extra).poison()
    semkv_assign_precision(cache, to_dev(S[:, :, :T0].copy()), T0, p)
    semkv_quantize_pack(cache, to_dev(K[:, :, :T0].copy()), to_dev(V[:, :, :T0].copy()), T0)
    for t in range(T0, T0 + steps):
        semkv_append_token(cache, to_dev(K[:, :, t].copy()), to_dev(V[:, :, t].copy()), to_dev(S[:, :, t].copy()))
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
    semkv_decode_attention(cache, to_dev(q), sm_scale(), out, cache.workspace())
    bufs = fetch(cache)
    status = cache.status()
    states = []
    for u in range(B * H):
        b, h = divmod(u, H)
        bm, rk, nh, tau, _ = oracle.select(S[b, h, :T0], p)
        hi, lo, _ = oracle.quantize_pack_unit(K[b, h, :T0].view(np.uint16), V[b, h, :T0].view(np.uint16), bm, G,
                                              L_hi, L_lo, cache.cap_hi // 128, cache.cap_lo // 128)
        st = oracle.UnitState(cache.T_cap, bm, rk, nh, T0 - nh, tau, hi, lo)
        ost = 0
        for t in range(T0, T0 + steps):
            ost |= oracle.append_unit(st, K[b, h, t].view(np.uint16), V[b, h, t].view(np.uint16), S[b, h, t], G,
                                      L_hi, L_lo)
        states.append((st, ost))
    return cache, bufs, status, out.cpu().numpy(), states, (K, V, S, q)


@pytest.mark.parametrize("p,L_hi,L_lo,G", [(0.25, 8, 5, 64), (0.5, 6, 5, 128), (0.1, 16, 3, 32)])
def test_append_matches_oracle_in_lockstep(p, L_hi, L_lo, G):
    import oracle

    B, H, Hq, T0, steps = 2, 2, 8, 300, 200
    cache, bufs, status, out, states, (K, V, S, q) = _append_lockstep(B, H, Hq, T0, steps, G, L_hi, L_lo, p, 9,
                                                                       extra=256)
    assert status == 0
    T = T0 + steps
    g = Hq // H
    for u, (st, ost) in enumerate(states):
        assert ost == 0
        gu = unit_views(cache, bufs, u)
        o = {"bitmap": st.bitmap, "rank": st.rank, "n_hi": st.n_hi, "tau": st.tau, "hi": st.hi, "lo": st.lo}
        compare_state(gu, o, T, L_hi, L_lo, where=f"unit {u}", strict_tail=False)
        b, h = divmod(u, H)
        Kh, Vh = oracle.dequantize_unit(T, 128, G, L_hi, L_lo, st.bitmap, st.hi, st.lo)
        ref = oracle.attention_fp64(q[b, h * g:(h + 1) * g].view(np.uint16), Kh, Vh, sm_scale())
        ma, rl = attention_errors(out[b, h * g:(h + 1) * g], ref)
        assert ma <= ATOL and rl <= RTOL_L2


def test_append_overflow_sets_status_and_keeps_state():
    B, H, Hq, T0, steps = 1, 1, 4, 120, 20  # lo segment: cap 128 slots; p = 0 so every token goes lo
    cache, bufs, status, out, states, _ = _append_lockstep(B, H, Hq, T0, steps, 64, 8, 5, 0.0, 4, extra=0)
    assert status & 4
    gu = unit_views(cache, bufs, 0)
    assert gu["n_lo"] == 128 and gu["n_hi"] == 0
    st, ost = states[0]
    assert ost & 4 and st.n_lo == 128
    compare_state(gu, {"bitmap": st.bitmap, "rank": st.rank, "n_hi": 0, "tau": st.tau, "hi": st.hi, "lo": st.lo},
                  128, 8, 5, strict_tail=False)


def test_empty_unit_decodes_to_zero():
    import torch

    from mixed_precision_kv_semkv_b200 import SemkvCache, semkv_assign_precision, semkv_decode_attention

    cache = SemkvCache(1, 2, 8, 64, 8, 5, 128, 128, 128)
    semkv_assign_precision(cache, to_dev(np.zeros((1, 2, 1), np.float32)), 0, 0.5)
    out = torch.full((1, 8, 128), 7.0, device="cuda")
    semkv_decode_attention(cache, to_dev(np.ones((1, 8, 128), np.float16)), 0.1, out, cache.workspace())
    assert not out.cpu().numpy().any()
