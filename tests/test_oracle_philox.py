"""Pins of the oracle's Philox4x32-10 and of its 24-bit uniforms (no GPU)."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from conftest import golden_path, ROOT
from oracle.philox import philox4x32_10, uniform


def _kat():
    rows = []
    for line in open(golden_path("philox4x32_10_kat.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        w = [int(t, 16) for t in line.split()]
        rows.append((w[:4], w[4:6], w[6:]))
    return rows


def test_known_answers():
    for ctr, key, want in _kat():
        got = philox4x32_10([np.uint64(c) for c in ctr], [np.uint64(k) for k in key])
        assert [int(g) for g in got] == want


def test_against_torch_engine(tmp_path):
    """Random counters/keys against PyTorch's independent Philox engine."""
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no g++")
    import torch.utils.cpp_extension as ext
    inc = ext.include_paths()
    exe = tmp_path / "philox_ref"
    cmd = [gxx, "-std=c++17", "-O1", os.path.join(ROOT, "tests", "philox_torch_ref.cpp"),
           "-o", str(exe)] + [f"-I{p}" for p in inc]
    subprocess.run(cmd, check=True, capture_output=True)
    rng = np.random.default_rng(5)
    ctr = rng.integers(0, 2 ** 32, size=(200, 4), dtype=np.uint64)
    key = rng.integers(0, 2 ** 32, size=(200, 2), dtype=np.uint64)
    inp = "\n".join(" ".join(f"{int(v):08x}" for v in list(c) + list(k)) for c, k in zip(ctr, key))
    res = subprocess.run([str(exe)], input=inp, capture_output=True, text=True, check=True)
    want = np.array([[int(t, 16) for t in line.split()] for line in res.stdout.strip().splitlines()])
    got = philox4x32_10([ctr[:, i] for i in range(4)], [key[:, 0], key[:, 1]])
    assert np.array_equal(np.stack([np.asarray(g) for g in got], 1).astype(np.int64), want)


def test_uniform_packing():
    # counter (request, purpose<<24 | position, lo32(round), hi32(round)), key (lo32, hi32 of seed)
    assert uniform(0, 0, 0, 0, 0) == 0x6627E8 / 2 ** 24
    ctr, key, want = _kat()[2]
    seed = key[0] | (key[1] << 32)
    rnd = ctr[2] | (ctr[3] << 32)
    purpose, pos = ctr[1] >> 24, ctr[1] & 0xFFFFFF
    assert uniform(seed, ctr[0], pos, purpose, rnd) == (want[0] >> 8) / 2 ** 24


def test_uniform_range_and_distinct_streams():
    u = uniform(1234, np.arange(100000), 3, 1, 7)
    assert u.min() >= 0.0 and u.max() < 1.0
    # 24-bit grid, exact in fp32
    assert np.all(u * 2 ** 24 == np.floor(u * 2 ** 24))
    assert np.all(u.astype(np.float32).astype(np.float64) == u)
    assert abs(u.mean() - 0.5) < 5 * (1 / np.sqrt(12 * len(u)))
    v = uniform(1234, np.arange(100000), 3, 2, 7)
    assert np.mean(u == v) < 1e-3
