"""The seeded input generator (the one module the CUDA path and the oracle share): the same seed
gives the same bytes, shapes and dtypes are the workloads', and the Zipf scores are a permutation of
r^-a normalised to sum 1, as documented."""
import numpy as np

from mixed_precision_kv_semkv_b200 import synth


def test_same_seed_same_bytes_other_seed_other_bytes():
    w = synth.WORKLOADS["tiny"]
    a = synth.layer_cpu(w, 3, T=300)
    b = synth.layer_cpu(w, 3, T=300)
    c = synth.layer_cpu(w, 4, T=300)
    for k in ("K", "V", "scores", "q"):
        assert a[k].tobytes() == b[k].tobytes(), k
        assert a[k].tobytes() != c[k].tobytes(), k
    assert a["K"].shape == (1, 1, 300, 128) and a["K"].dtype == np.float16
    assert a["q"].shape == (1, 4, 128) and a["q"].dtype == np.float16
    assert a["scores"].shape == (1, 1, 300) and a["scores"].dtype == np.float32


def test_zipf_scores_are_a_permutation_of_the_power_law():
    T, a = 500, 1.1
    s = synth.zipf_scores_cpu(a, T, 3, 7)
    ref = np.arange(1, T + 1, dtype=np.float64) ** -a
    ref /= ref.sum()
    for u in range(s.shape[0]):
        row = np.sort(s[u].astype(np.float64))[::-1]
        assert np.allclose(row, ref, rtol=1e-6, atol=0)
        assert len(np.unique(s[u])) == T  # no ties


def test_p_for_ratio_kv_rejects_bad_arguments(semkv):
    import pytest

    for args, code in (((128, 64, 8, 5, 1, 2, 4.0), 2), ((128, 64, 8, 5, 4, 300, 4.0), 2),
                       ((128, 64, 8, 5, 4, 2, 0.0), 1), ((128, 48, 8, 5, 4, 2, 4.0), 1)):
        with pytest.raises(semkv.SemkvError) as e:
            semkv.semkv_p_for_ratio_kv(*args)
        assert e.value.code == code, args


def test_generated_tokens_share_the_prefill_channel_scales():
    """The GPU-path generator (run here on the CPU device) draws generated k, v with the prefill's
    per-channel scales: divided by those scales, both the prefill rows and the generated rows have
    unit spread in every channel, while the raw channels do not."""
    import torch

    w = synth.WORKLOADS["llama8b_1L"]
    d = synth.layer_gpu(w, 5, layer=2, device="cpu", T=4096)
    sk, sv = synth.prefill_channel_scales_gpu(w, 5, layer=2, device="cpu")
    gen = synth.gen_steps_gpu(w, d["K"], 5, 2, steps=4096, device="cpu")
    assert gen["k"].shape == (4096, 1, 8, 128) and gen["k"].dtype == torch.float16
    for x, s in ((d["K"].float(), sk), (d["V"].float(), sv)):
        r = (x / s).std(dim=2)  # [B][H][D] over the prefill tokens
        assert torch.allclose(r, torch.ones_like(r), atol=0.08)
    for x, s in ((gen["k"].float(), sk.reshape(1, 1, 8, 128)), (gen["v"].float(), sv.reshape(1, 1, 8, 128))):
        r = (x / s).std(dim=0)  # over the generated tokens
        assert torch.allclose(r, torch.ones_like(r), atol=0.08)
        raw = x.std(dim=0)
        assert raw.max() / raw.min() > 2.0  # the channel scales are really there


def test_outlier_workload_has_no_channel_scales():
    assert synth.prefill_channel_scales_gpu(synth.WORKLOADS["tiny"], 0, device="cpu") == (None, None)
