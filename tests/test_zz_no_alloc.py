"""The allocation-free decode entry point (semkv_decode_attention_noalloc).

It serves callers that cannot allocate device memory when they decode -- for example a plugin in
a server whose process has given all device memory to its own pool allocator.  Instead of a
caller-provided workspace it keeps the split-K partials in a fixed array inside the library.
These tests call it through the C ABI and check it against semkv_decode_attention (which takes a
workspace) on two calls in a row: the first over a larger cache, the second over a smaller cache
with other queries, so that partials left in the array by the first call would show up in the
second call's output.  The two entry points run the same kernels on the same inputs, so their
outputs must agree bit for bit (that is within the attention tolerance the other tests use, and
stricter).  The file is named so that pytest collects it last.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _prefill(w, seed, T):
    import torch

    from mixed_precision_kv_semkv_b200 import SemkvCache, semkv_assign_precision, semkv_quantize_pack, synth

    d = synth.layer_cpu(w, seed, T=T)
    K, V, S, q = (torch.from_numpy(d[n]).cuda() for n in ("K", "V", "scores", "q"))
    cache = SemkvCache.for_prefill(w.B, w.H, w.Hq, w.G, w.L_hi, w.L_lo, T, w.p)
    semkv_assign_precision(cache, S, T, w.p)
    semkv_quantize_pack(cache, K, V, T)
    return cache, q


def test_noalloc_decode_matches_workspace_decode_twice():
    import torch

    from mixed_precision_kv_semkv_b200 import (build, semkv_decode_attention, semkv_decode_attention_noalloc,
                                               synth)

    build.build()
    w = synth.WORKLOADS["llama8b_1L"]
    for seed, T in ((3, 6000), (4, 1500)):  # a larger cache, then a smaller one with other queries
        cache, q = _prefill(w, seed, T)
        ref = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
        semkv_decode_attention(cache, q, synth.sm_scale(), ref, cache.workspace())
        out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.float32, device="cuda")
        semkv_decode_attention_noalloc(cache, q, synth.sm_scale(), out)
        got, want = out.cpu().numpy(), ref.cpu().numpy()
        assert np.isfinite(want).all()
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (T, float(np.abs(got - want).max()))
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
