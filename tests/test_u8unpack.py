"""The byte unpack of the integer tensor-core decode (csrc/i8unpack.cuh), checked on the CPU.

Rows of random codes (and the all-0 and all-(L-1) rows) are packed into base-L words by the
oracle's packer (SemKV page, Abstract: codes on L-level grids, k(L) per 32-bit word); the header's
unpack, compiled for the host, must put code row_index(pos) at every operand byte pos, row_pos must
be its inverse, every table index must stay inside the table, and words that are not valid packings
(any 32-bit pattern, as stale slots hold) must still unpack without an out-of-range index."""
import os
import shutil
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    out = str(tmp_path_factory.mktemp("u8") / "u8unpack")
    subprocess.run([nvcc, "-std=c++17", "-O1", "-o", out, os.path.join(HERE, "host", "u8unpack_main.cu")],
                   check=True, capture_output=True)
    return out


def _run(driver, L, words):
    inp = f"{L} {len(words)}\n" + "\n".join(" ".join(str(int(x)) for x in row) for row in words) + "\n"
    r = subprocess.run([driver], input=inp, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout[-500:] + r.stderr[-500:]
    lines = r.stdout.strip().splitlines()
    rows = np.array([[int(x) for x in ln.split()] for ln in lines[: len(words)]], dtype=np.int64)
    idx = np.array([int(x) for x in lines[len(words)].split()])
    pos = np.array([int(x) for x in lines[len(words) + 1].split()])
    return rows, idx, pos


@pytest.mark.parametrize("L", [4, 5, 6, 8, 16])
def test_unpack_places_every_code(orc, driver, L):
    k = orc.radix_digits(L)
    W = -(-128 // k)
    r = np.random.default_rng(L)
    codes = [r.integers(0, L, 128) for _ in range(40)] + [np.zeros(128, np.int64), np.full(128, L - 1)]
    words = []
    for c in codes:
        padded = np.zeros(W * k, np.uint8)
        padded[:128] = c
        words.append([orc.pack_word(padded[j * k:(j + 1) * k], L) for j in range(W)])
    rows, idx, pos = _run(driver, L, words)
    assert sorted(idx.tolist()) == list(range(128))          # a permutation of the row
    assert np.array_equal(pos[idx], np.arange(128))          # row_pos inverts row_index
    for c, got in zip(codes, rows):
        assert np.array_equal(got, np.asarray(c)[idx])


@pytest.mark.parametrize("L", [5, 6, 8])
def test_any_word_stays_inside_the_table(driver, L):
    r = np.random.default_rng(100 + L)
    k = {5: 13, 6: 12, 8: 10}[L]
    W = -(-128 // k)
    words = r.integers(0, 2 ** 32, size=(60, W), dtype=np.uint64).tolist()
    words.append([2 ** 32 - 1] * W)
    rows, _, _ = _run(driver, L, words)
    assert rows.max() < L  # every byte is still a digit
