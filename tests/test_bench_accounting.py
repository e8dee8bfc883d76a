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
    assert d["config"]["workload"] == bench.workload_config(synth.WORKLOADS["llama8b_1L"], 1)["workload"]
