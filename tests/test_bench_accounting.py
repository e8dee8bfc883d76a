"""The algorithmic bytes bench.py divides by (the `value` and the roofline's `achieved`), checked
against the closed forms of the measurement section worked out by hand for the Llama-3.1-8B-shaped
layer: B1 H8 Hq32 T32768 D128, G64, L 8/5, p 0.25 (n_hi 8192, n_lo 24576 per unit)."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from mixed_precision_kv_semkv_b200 import synth  # noqa: E402


def test_radix_words_agree_with_the_oracle(orc):
    for L in range(2, 257):
        assert bench.radix_words(L) == orc.words_per_row(L, 128) == orc.words_per_tile_column(L)


def test_decode_and_quantize_bytes_by_hand():
    w = synth.WORKLOADS["llama8b_1L"]
    nb = bench.alg_bytes(w, 32768, 8192)
    # one token's K + V record: words (13 at L 8, 10 at L 5) and two fp16 scale/zero pairs, twice
    rec_hi, rec_lo = 2 * (4 * 13 + 4 * 2), 2 * (4 * 10 + 4 * 2)  # 120 and 96 bytes
    cache = 8 * (8192 * rec_hi + 24576 * rec_lo)                  # 26,738,688
    assert nb["cache"] == cache == 26_738_688
    assert nb["decode"] == cache + 1 * 32 * 128 * 2               # + the fp16 queries
    bitmap_rank = 8 * 2 * 4 * (32768 // 32)
    assert nb["quantize"] == 8 * 32768 * 128 * 2 * 2 + bitmap_rank + cache == 161_021_952
    assert nb["select"] == 8 * 4 * 32768 + bitmap_rank
    # with one appended token per unit, all on the coarse grid
    nb1 = bench.alg_bytes(w, 32768, 8192, new_hi=0, appended=True)
    assert nb1["decode"] == nb["decode"] + 8 * rec_lo
    assert nb1["append"] == 8 * (128 * 2 * 2 + 4) + 8 * rec_lo


def test_v_level_bytes_by_hand():
    # V on 4 (16 codes per word: 8 words per 128-slot column) and 2 levels (32: 4 words): per token
    # hi 52 (K) + 32 (V) + 16 (scale/zero) = 100 bytes, lo 40 + 16 + 16 = 72 bytes
    w = synth.WORKLOADS["llama8b_1L"]
    nb = bench.alg_bytes(w, 32768, 8192, v_levels=(4, 2))
    assert nb["cache"] == 8 * (8192 * 100 + 24576 * 72)


def test_reference_arm_prints_its_contract_line():
    """`bench.py --impl reference` (the oracle on the host, a bounded sample) prints one JSON line
    with the keys of the contract and the same config as the GPU arm's."""
    import json
    import subprocess

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == bench.workload_config(synth.WORKLOADS["gen"], 1)["workload"]
    assert d["cpu_baseline"]["cores"] >= 1


def test_generation_step_bytes_by_hand():
    """Two layers of the generation workload's shape (16 x 8 = 128 units), 4 steps: layer 0 puts 3
    of its 512 new tokens on the fine grid, layer 1 none.  Per step j the decode reads every record
    of T0 + j tokens per unit plus the queries; the append reads k, v rows and the score and writes
    one record per unit."""
    w = synth.WORKLOADS["gen"]
    U, steps = 128, 4
    rec_hi, rec_lo = 120, 96  # L 8 and L 5 at G64 (see test_decode_and_quantize_bytes_by_hand)
    nh0, nl0 = [U * 8192, U * 8192], [U * 24576, U * 24576]
    nh1, nl1 = [nh0[0] + 3, nh0[1]], [nl0[0] + U * steps - 3, nl0[1] + U * steps]
    nb = bench.gen_steps_bytes(w, nh0, nl0, nh1, nl1, steps)
    q = 16 * 32 * 128 * 2
    dec = 0.0
    for j in range(1, steps + 1):
        for layer, dh in ((0, 3), (1, 0)):
            dec += (nh0[layer] + j * dh / steps) * rec_hi + (nl0[layer] + j * (U * steps - dh) / steps) * rec_lo + q
    assert nb["decode"] == dec
    app = 2 * steps * U * (128 * 2 * 2 + 4) + 3 * rec_hi + (2 * U * steps - 3) * rec_lo
    assert nb["append"] == app and nb["total"] == dec + app


# storage reduction against fp16 of the precision sweep's 45 points, from the closed form of the
# physical bits per value worked out by hand:
#   bits(p) = p B(L_hi) + (1 - p) B(L_lo) + 32/G + 1/256,  B(L) = 32 ceil(128/k(L)) / 128
# with k(5, 6, 8, 16) = 13, 12, 10, 8 codes per word (10, 11, 13, 16 words: B = 2.5, 2.75, 3.25, 4),
# ratio = 16 / bits(p), rounded to 3 decimals (one row per level pair, G = 32 / 64 / 128 per p).
SWEEP_RATIOS = {
    (6, 5): {0.0: (4.566, 5.326, 5.810), 0.25: (4.486, 5.218, 5.681), 0.5: (4.409, 5.114, 5.558),
             0.75: (4.334, 5.013, 5.440), 1.0: (4.262, 4.917, 5.326)},
    (8, 6): {0.0: (4.262, 4.917, 5.326), 0.25: (4.125, 4.735, 5.114), 0.5: (3.996, 4.566, 4.917),
             0.75: (3.875, 4.409, 4.735), 1.0: (3.761, 4.262, 4.566)},
    (16, 8): {0.0: (3.761, 4.262, 4.566), 0.25: (3.602, 4.059, 4.334), 0.5: (3.457, 3.875, 4.125),
              0.75: (3.322, 3.707, 3.935), 1.0: (3.198, 3.552, 3.761)},
}


def test_sweep_storage_ratios_equal_the_closed_form(semkv):
    """The ratio the bench prints per sweep point (from the library's buffer sizes for the sweep's
    cache: batch 8, 8 KV heads, T 32768) equals the closed form at all 45 points."""
    w = synth.WORKLOADS["mistral_sweep"]
    n = 0
    for (Lh, Ll), rows in SWEEP_RATIOS.items():
        for p, per_g in rows.items():
            for G, want in zip((32, 64, 128), per_g):
                got = bench.storage_ratio(128, G, Lh, Ll, p, w.T, B=w.B, H=w.H)
                assert round(got, 3) == want, (Lh, Ll, p, G, got, want)
                n += 1
    assert n == 45 == len(synth.SWEEP_PAIRS) * len(synth.SWEEP_P) * len(synth.SWEEP_G)
