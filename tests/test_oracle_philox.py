"""Oracle pins: the Philox4x32-10 stream (stochastic rounding and RHT signs).

The oracle implements Philox4x32-10 from Salmon et al., "Parallel Random
Numbers: As Easy as 1, 2, 3" (SC'11).  It is pinned here to an independent
implementation, PyTorch's header-only at::philox_engine, compiled on the host,
and to statistical properties of the words.
"""
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def build_torch_philox(out_dir: str) -> str:
    """Compile the helper that prints PyTorch's Philox4x32-10 blocks."""
    import torch
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    src = os.path.join(HERE, "helpers", "torch_philox.cpp")
    exe = os.path.join(out_dir, "torch_philox")
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", inc, src, "-o", exe], check=True)
    return exe


@pytest.fixture(scope="module")
def torch_philox():
    # the mutation tests compile the helper once and pass it in
    exe = os.environ.get("MXFP4_TORCH_PHILOX") or build_torch_philox(tempfile.mkdtemp())

    def run(triples):
        inp = "".join(f"{s} {q} {o}\n" for s, q, o in triples)
        out = subprocess.run([exe], input=inp, capture_output=True, text=True, check=True).stdout
        return [[int(v) for v in line.split()] for line in out.strip().splitlines()]
    return run


def test_philox_blocks_match_torch_engine(torch_philox):
    g = np.random.default_rng(99)
    triples = [(0, 0, 0), (1, 0, 0), (42, 0, 0), (0xFFFFFFFFFFFFFFFF, 0, 0), (42, 0, 1), (42, 0, 2 ** 32 + 5)]
    triples += [(int(s), int(q), int(o)) for s, q, o in
                zip(g.integers(0, 2 ** 63, 200), g.integers(0, 2 ** 63, 200), g.integers(0, 2 ** 63, 200))]
    ref = torch_philox(triples)
    for (seed, subseq, off), words in zip(triples, ref):
        ctr = [off & 0xFFFFFFFF, off >> 32, subseq & 0xFFFFFFFF, subseq >> 32]
        key = [seed & 0xFFFFFFFF, seed >> 32]
        assert oracle.philox4x32_10(ctr, key) == words


def test_sr_stream_indexing_matches_torch_engine(torch_philox):
    # element g uses word g % 4 of the block with counter (g/4, 0): torch's
    # engine with subsequence 0 and offset g/4.
    seed = 42
    gs = [0, 1, 2, 3, 4, 5, 1023, 2 ** 32 * 4 + 7, 11796480 - 1]
    ref = torch_philox([(seed, 0, g >> 2) for g in gs])
    for g, words in zip(gs, ref):
        assert oracle.sr_word(seed, g) == words[g & 3]
    words = oracle.sr_words(seed, 1000, 64)
    assert all(int(words[i]) == oracle.sr_word(seed, 1000 + i) for i in range(64))


def test_rht_sign_mask_matches_torch_engine(torch_philox):
    for seed in (0, 42, 7, 2 ** 40 + 3):
        ref = torch_philox([(seed, 0x52485400 << 32, 0)])[0]
        assert oracle.rht_sign_mask(seed) == ref[0]


def test_philox_words_are_balanced():
    n = 1 << 20
    w = oracle.sr_words(2024, 0, n)
    bits = np.unpackbits(w.view(np.uint8)).reshape(n, 32)
    p = bits.mean(axis=0)
    # each bit is Bernoulli(1/2): 6 sigma = 6 * 0.5 / sqrt(n)
    assert np.all(np.abs(p - 0.5) < 6 * 0.5 / np.sqrt(n))
    # chi-squared on the top byte (255 dof): mean 255, sd ~22.6; 8 sd margin
    counts = np.bincount((w >> 24).astype(np.int64), minlength=256)
    exp = n / 256
    chi2 = float(((counts - exp) ** 2 / exp).sum())
    assert abs(chi2 - 255) < 8 * np.sqrt(2 * 255)
