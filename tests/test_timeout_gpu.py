"""Bounded waits give up and report SEMKV_STATUS_TIMEOUT without hanging the GPU.

semkv_selftest_wait_timeout launches one warp whose mbarrier wait nothing completes (one of two
expected arrivals), with a short test bound; the kernel must return, set the status bit and free
the tensor memory it held, and the device must stay usable: a decode launched right after it (whose
kernels allocate all of an SM's tensor memory) still matches the oracle-checked path's result.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("use_tmem", [False, True])
def test_wait_gives_up_and_sets_timeout(use_tmem):
    import torch

    from mixed_precision_kv_semkv_b200 import _lib, build, semkv_selftest_wait_timeout

    build.build()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    semkv_selftest_wait_timeout(status, tests=16, use_tmem=use_tmem)
    torch.cuda.synchronize()  # raises if the kernel faulted
    assert int(status.item()) == _lib.STATUS_TIMEOUT


def test_device_usable_after_timeouts():
    import torch

    from mixed_precision_kv_semkv_b200 import (SemkvCache, build, semkv_assign_precision, semkv_decode_attention,
                                               semkv_quantize_pack, semkv_selftest_wait_timeout, synth)

    build.build()
    w = synth.WORKLOADS["llama8b_1L"]
    d = synth.layer_cpu(w, 5, T=3000)
    K, V, S, q = (torch.from_numpy(d[n]).cuda() for n in ("K", "V", "scores", "q"))
    cache = SemkvCache.for_prefill(w.B, w.H, w.Hq, w.G, w.L_hi, w.L_lo, 3000, w.p)
    semkv_assign_precision(cache, S, 3000, w.p)
    semkv_quantize_pack(cache, K, V, 3000)
    ref = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    semkv_decode_attention(cache, q, synth.sm_scale(), ref, cache.workspace())
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(4):  # many SMs' worth of tensor memory allocated and freed around timed-out waits
        semkv_selftest_wait_timeout(status, tests=4, use_tmem=True)
    out = torch.full_like(ref, float("nan"))
    semkv_decode_attention(cache, q, synth.sm_scale(), out, cache.workspace())
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.cpu().numpy().view(np.uint32))
    assert cache.status() == 0

