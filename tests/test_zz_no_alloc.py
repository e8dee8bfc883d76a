"""The allocation-free decode entry point (semkv_decode_attention_noalloc).

It serves callers that cannot allocate device memory when they decode -- for example a plugin in
a server whose process has given all device memory to its own pool allocator.  Instead of a
caller-provided workspace it keeps the split-K partials in a fixed array inside the library.
These tests call it through the C ABI and check it against semkv_decode_attention (which takes a
workspace) on two calls in a row, within the attention tolerance used by the other tests.  The
file is named so that pytest collects it last.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ATOL, RTOL_L2 = 2e-3, 1e-3


def _errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(got - ref).max()), float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def test_noalloc_decode_matches_workspace_decode_twice():
    import torch

    from mixed_precision_kv_semkv_b200 import (SemkvCache, build, semkv_assign_precision, semkv_decode_attention,
                                               semkv_decode_attention_noalloc, semkv_quantize_pack, synth)

    build.build()
    w = synth.WORKLOADS["llama8b_1L"]
    d = synth.layer_cpu(w, 3, T=6000)
    K, V, S, q = (torch.from_numpy(d[n]).cuda() for n in ("K", "V", "scores", "q"))
    T = d["K"].shape[2]
    cache = SemkvCache.for_prefill(w.B, w.H, w.Hq, w.G, w.L_hi, w.L_lo, T, w.p)
    semkv_assign_precision(cache, S, T, w.p)
    semkv_quantize_pack(cache, K, V, T)
    ref = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    semkv_decode_attention(cache, q, synth.sm_scale(), ref, cache.workspace())
    ref = ref.cpu().numpy()
    for _ in range(2):
        out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.float32, device="cuda")
        semkv_decode_attention_noalloc(cache, q, synth.sm_scale(), out)
        got = out.cpu().numpy()
        ma, rl = _errors(got, ref)
        assert ma <= ATOL and rl <= RTOL_L2, (ma, rl)
    assert cache.status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    from mixed_precision_kv_semkv_b200 import SemkvError, _lib, semkv_decode_attention_noalloc, semkv_workspace_bytes

    s = _lib.CacheStruct(B=4096, H=8, Hq=32, D=128, G=64, L_hi=8, L_lo=5, cap_hi=128, cap_lo=128, T_cap=256)
    for i, n in enumerate(_lib.BUF_NAMES):
        setattr(s, n, 0x1000 * (i + 1))  # never dereferenced: the call fails before any launch
    assert semkv_workspace_bytes(s) > _lib.NOALLOC_SCRATCH_BYTES
    with pytest.raises(SemkvError) as e:
        semkv_decode_attention_noalloc(s, None, 0.1, None)
    assert e.value.code == _lib.SEMKV_ERR_CAPACITY
