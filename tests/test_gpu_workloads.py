"""Full-size runs of the other workloads (32-layer Llama-3.1-8B cache at T=131072, generation with
batch 16 and 256 appended tokens, the Mistral-7B-shaped precision sweep), each checked against the
oracle on sampled units: the same bit-exact state and the same attention tolerance as the small
parity tests.  Inputs are drawn on the GPU by the seeded generator; the sampled units' inputs are
copied to the host for the oracle."""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

from gpu_harness import ATOL, RTOL_L2, attention_errors, compare_state, fetch, unit_views  # noqa: E402


def _oracle_prefill(K16, V16, S, p, G, L_hi, L_lo, cache):
    import oracle

    bm, rk, nh, tau, st = oracle.select(S, p)
    hi, lo, st2 = oracle.quantize_pack_unit(K16, V16, bm, G, L_hi, L_lo, cache.cap_hi // 128, cache.cap_lo // 128)
    return {"bitmap": bm, "rank": rk, "n_hi": nh, "tau": tau, "hi": hi, "lo": lo, "status": st | st2}


def _check_unit_attention(out_u, q_u, state, T, G, L_hi, L_lo, scale):
    import oracle

    Kh, Vh = oracle.dequantize_unit(T, 128, G, L_hi, L_lo, state["bitmap"], state["hi"], state["lo"])
    ref = oracle.attention_fp64(q_u.view(np.uint16), Kh, Vh, scale)
    ma, rl = attention_errors(out_u, ref)
    assert ma <= ATOL and rl <= RTOL_L2, (ma, rl)
    return ma, rl


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_kv_semkv_b200 import build

    build.build()


def test_llama8b_32_layers_T131072_sampled():
    import torch

    from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_assign_precision, semkv_decode_attention,
                                               semkv_quantize_pack, synth)

    w = synth.WORKLOADS["llama8b_32L"]
    sampled = {0: 3, 17: 0, 31: 6}  # layer -> kv head checked against the oracle
    g = w.Hq // w.H
    for layer in range(w.layers):
        d = synth.layer_gpu(w, seed=0, layer=layer)
        cache = SemkvCache.for_prefill(w.B, w.H, w.Hq, w.G, w.L_hi, w.L_lo, w.T, w.p)
        semkv_assign_precision(cache, d["scores"], w.T, w.p)
        semkv_quantize_pack(cache, d["K"], d["V"], w.T)
        out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
        semkv_decode_attention(cache, d["q"], synth.sm_scale(), out, cache.workspace())
        torch.cuda.synchronize()
        assert cache.status() == 0
        if layer in sampled:
            h = sampled[layer]
            bufs = fetch(cache)
            K = d["K"][0, h].cpu().numpy().view(np.uint16)
            V = d["V"][0, h].cpu().numpy().view(np.uint16)
            S = d["scores"][0, h].cpu().numpy()
            o = _oracle_prefill(K, V, S, w.p, w.G, w.L_hi, w.L_lo, cache)
            assert o["status"] == 0
            compare_state(unit_views(cache, bufs, h), o, w.T, w.L_hi, w.L_lo, where=f"layer {layer} head {h}")
            _check_unit_attention(out[0, h * g:(h + 1) * g].cpu().numpy(), d["q"][0, h * g:(h + 1) * g].cpu().numpy(),
                                  o, w.T, w.G, w.L_hi, w.L_lo, synth.sm_scale())
        del d, cache


def test_generation_batch16_256_steps_sampled():
    import torch

    import oracle
    from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_append_token, semkv_assign_precision,
                                               semkv_decode_attention, semkv_quantize_pack, synth)

    w = synth.WORKLOADS["gen"]
    g = w.Hq // w.H
    sampled = {(2, 5, 3), (29, 11, 7)}  # (layer, batch row, kv head)
    check_steps = (0, 127, w.steps - 1)
    for layer in range(w.layers):
        d = synth.layer_gpu(w, seed=1, layer=layer)
        st = synth.gen_steps_gpu(w, d["K"], seed=1, layer=layer, steps=w.steps)
        cache = SemkvCache.for_prefill(w.B, w.H, w.Hq, w.G, w.L_hi, w.L_lo, w.T, w.p, extra=w.steps).poison()
        cache.clear_status()
        semkv_assign_precision(cache, d["scores"], w.T, w.p)
        semkv_quantize_pack(cache, d["K"], d["V"], w.T)
        ws = cache.workspace()
        out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
        outs = {}
        for s in range(w.steps):
            semkv_append_token(cache, st["k"][s], st["v"][s], st["scores"][s])
            semkv_decode_attention(cache, st["q"][s], synth.sm_scale(), out, ws)
            if s in check_steps:
                outs[s] = out.cpu().numpy()
        torch.cuda.synchronize()
        assert cache.status() == 0
        for (lyr, b, h) in sampled:
            if lyr != layer:
                continue
            u = b * w.H + h
            K = d["K"][b, h].cpu().numpy().view(np.uint16)
            V = d["V"][b, h].cpu().numpy().view(np.uint16)
            S = d["scores"][b, h].cpu().numpy()
            o = _oracle_prefill(K, V, S, w.p, w.G, w.L_hi, w.L_lo, cache)
            state = oracle.UnitState(cache.T_cap, o["bitmap"], o["rank"], o["n_hi"], w.T - o["n_hi"], o["tau"],
                                     o["hi"], o["lo"])
            kn = st["k"][:, b, h].cpu().numpy().view(np.uint16)
            vn = st["v"][:, b, h].cpu().numpy().view(np.uint16)
            sn = st["scores"][:, b, h].cpu().numpy()
            qn = st["q"][:, b, h * g:(h + 1) * g].cpu().numpy()
            for s in range(w.steps):
                assert oracle.append_unit(state, kn[s], vn[s], sn[s], w.G, w.L_hi, w.L_lo) == 0
                if s in check_steps:
                    ost = {"bitmap": state.bitmap, "rank": state.rank, "n_hi": state.n_hi, "tau": state.tau,
                           "hi": state.hi, "lo": state.lo}
                    _check_unit_attention(outs[s][b, h * g:(h + 1) * g], qn[s], ost, w.T + s + 1, w.G, w.L_hi,
                                          w.L_lo, synth.sm_scale())
            bufs = fetch(cache)
            ost = {"bitmap": state.bitmap, "rank": state.rank, "n_hi": state.n_hi, "tau": state.tau,
                   "hi": state.hi, "lo": state.lo}
            compare_state(unit_views(cache, bufs, u), ost, w.T + w.steps, w.L_hi, w.L_lo,
                          where=f"layer {layer} unit {u}", strict_tail=False)
        del d, st, cache


def test_mistral_sweep_45_points_sampled():
    import torch

    import oracle
    from mixed_precision_kv_semkv_b200 import (SemkvCache, semkv_assign_precision, semkv_decode_attention,
                                               semkv_quantize_pack, synth)

    w = synth.WORKLOADS["mistral_sweep"]
    g = w.Hq // w.H
    data = [synth.layer_gpu(w, seed=2, layer=layer) for layer in (0, 31)]  # two layers' inputs, reused per point
    i = 0
    for (L_hi, L_lo) in synth.SWEEP_PAIRS:
        for p in synth.SWEEP_P:
            for G in synth.SWEEP_G:
                d = data[i % 2]
                cache = SemkvCache.for_prefill(w.B, w.H, w.Hq, G, L_hi, L_lo, w.T, p)
                semkv_assign_precision(cache, d["scores"], w.T, p)
                semkv_quantize_pack(cache, d["K"], d["V"], w.T)
                out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
                semkv_decode_attention(cache, d["q"], synth.sm_scale(), out, cache.workspace())
                torch.cuda.synchronize()
                assert cache.status() == 0
                # storage ratio against fp16: the packed cache's bytes for full tiles vs the closed form
                nh = oracle.n_hi(p, w.T)
                words = lambda L: math.ceil(128 / oracle.radix_digits(L))  # noqa: E731
                closed = (nh * (32 * words(L_hi)) + (w.T - nh) * (32 * words(L_lo))) / (w.T * 128) + 32 / G + 1 / 256
                bits = oracle.storage_bits_per_value(128, G, L_hi, L_lo, nh / w.T)
                assert abs(bits - closed) < 1e-9 and 16 / bits > 3.0
                # one sampled unit per point against the oracle
                b, h = i % w.B, (3 * i) % w.H
                u = b * w.H + h
                K = d["K"][b, h].cpu().numpy().view(np.uint16)
                V = d["V"][b, h].cpu().numpy().view(np.uint16)
                S = d["scores"][b, h].cpu().numpy()
                o = _oracle_prefill(K, V, S, p, G, L_hi, L_lo, cache)
                compare_state(unit_views(cache, fetch(cache), u), o, w.T, L_hi, L_lo, where=f"point {i}")
                _check_unit_attention(out[b, h * g:(h + 1) * g].cpu().numpy(), d["q"][b, h * g:(h + 1) * g].cpu().numpy(),
                                      o, w.T, G, L_hi, L_lo, synth.sm_scale())
                del cache
                i += 1
    assert i == 45
