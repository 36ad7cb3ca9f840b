"""Structured rotation D1 H D2 H D3 / 128 (tq_build_hadamard_rotation and the input generator):
the SplitMix64 sign source against its published outputs, exact orthogonality and fp16-exact
entries, the product against scipy's Sylvester Hadamard matrix, the C builder against the input
generator, and the oracle's quantization MSE with this rotation against the pages' figures and
against the dense Haar rotation.  CPU only (the C builder runs on the host)."""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.linalg import hadamard

import decode_attention_11_b200 as tq
import workloads as W
from oracle import tq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")


def test_splitmix64_published_outputs():
    # the first three outputs of SplitMix64 started at state 0, as published with the generator
    assert [W.splitmix64(0, n) for n in range(3)] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4,
                                                      0x06C45D188009454F]


@pytest.mark.parametrize("seed", [0, 1001, (1 << 64) - 1])
def test_hadamard_rotation_exact(seed):
    P = W.make_hadamard_rotation(seed).astype(np.float64)
    assert np.array_equal(P @ P.T, np.eye(128))  # exact: entries are multiples of 1/64
    assert np.array_equal(P * 64, np.round(P * 64))
    assert np.array_equal(P.astype(np.float16).astype(np.float64), P)


def test_hadamard_rotation_is_the_stated_product():
    seed = 1001
    H = hadamard(128).astype(np.float64)
    D = [np.diag([1.0 if W.splitmix64(seed, 128 * k + i) % 2 == 0 else -1.0 for i in range(128)])
         for k in range(3)]
    P = D[0] @ H @ D[1] @ H @ D[2] / 128
    assert np.array_equal(P, W.make_hadamard_rotation(seed).astype(np.float64))
    # not a signed permutation: every output mixes many inputs
    assert np.min(np.sum(P != 0, axis=1)) >= 32


@pytest.mark.parametrize("seed", [0, 1001, 12345678901234567, (1 << 64) - 1])
def test_c_builder_matches_generator(seed):
    assert np.array_equal(tq.build_hadamard_rotation(seed), W.make_hadamard_rotation(seed))


def _normalized_mse(X, Pi, bits):
    r = O.quantize_vectors(X, Pi, bits)
    xh = (r["n"][:, None] / math.sqrt(128)) * O.codebook(bits).centroids[r["idx"]] @ Pi.astype(np.float64)
    return float(np.mean(np.sum((X - xh) ** 2, 1) / np.sum(X ** 2, 1)))


def test_pages_normalized_mse_with_hadamard_rotation():
    """Random-direction vectors: TQ3 0.034 and TQ4 0.009 at the printed precision, as with Haar."""
    with open(GOLDEN) as f:
        p = json.load(f)
    g = torch.Generator().manual_seed(7)
    X = torch.randn(40000, 128, generator=g, dtype=torch.float64).numpy()
    Pi = W.make_hadamard_rotation(1007)
    for bits, key in ((3, "tq3_normalized_mse"), (4, "tq4_normalized_mse")):
        mse = _normalized_mse(X, Pi, bits)
        assert abs(mse - p[key]["value"]) <= 0.5 * 10.0 ** -p[key]["printed_digits"], (bits, mse)


@pytest.mark.parametrize("name", ["single_head_4k", "llama3_8b_32k", "llama3_70b_16k_b16"])
def test_hadamard_mse_not_worse_than_haar_on_workload_keys(name):
    """Keys with outlier channels / heavy tails: the structured rotation spreads them at least as
    well as the dense one (normalized MSE within 2% or lower)."""
    w = W.CONFIGS[name]
    w = w.scaled(T=min(w.T, 1024), B=1)
    X = W.make_kv(w, "k").reshape(-1, 128).double().numpy()
    for bits in (3, 4):
        haar = _normalized_mse(X, W.make_rotation(1000 + w.seed), bits)
        had = _normalized_mse(X, W.make_hadamard_rotation(1000 + w.seed), bits)
        assert had <= 1.02 * haar, (name, bits, had, haar)
