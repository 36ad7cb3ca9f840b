"""CPU pins of the oracle's outlier-aware mixed-precision layout (3.5 bits: an outlier half of the
channels at 4 bits, the other half at 3).  Pages: tproger.ru, section on TheTom's llama.cpp fork
(turbo3 = 3.5-bit KV quantization, 4.6x vs FP16); ai-manual.ru M5 Max KV-cache benchmark
(per-layer outlier-aware 3/4-bit).  Each pin ties the mixed functions to something other than
their own formulas: the plain oracle run on each half, the pages' printed figures, brute force and
the QJL estimator's unbiasedness."""
import json
import math
import os

import numpy as np
import pytest

import workloads as W
from oracle import tq_oracle as O

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")))
BITS = (4, 3)


def _setup(n=300, seed=0):
    rng = np.random.default_rng(seed)
    oc = np.sort(rng.permutation(128)[:64])
    P = W.make_block_rotation(4242, oc).astype(np.float64)
    X = rng.standard_normal((n, 128)) * np.exp(0.5 * rng.standard_normal(128))
    return rng, oc, P, X


def test_block_rotation_structure():
    _, oc, P, _ = _setup()
    rest = np.setdiff1d(np.arange(128), oc)
    assert np.abs(P @ P.T - np.eye(128)).max() <= 1e-6
    assert np.all(P[:64][:, rest] == 0) and np.all(P[64:][:, oc] == 0)
    assert np.array_equal(P[:64][:, oc], W.make_rotation(4242, 64).astype(np.float64))
    assert np.array_equal(P[64:][:, rest], W.make_rotation(4243, 64).astype(np.float64))


def test_each_half_is_the_plain_method_on_its_channels():
    """The mixed codes of half O (R) equal the plain oracle's codes of the 64-dimensional problem
    on the outlier (other) channels with that half's rotation and bit width."""
    _, oc, P, X = _setup()
    rest = np.setdiff1d(np.arange(128), oc)
    mq = O.quantize_vectors_mixed(X, P, oc, *BITS)
    for g, (chans, bits) in enumerate(((oc, BITS[0]), (rest, BITS[1]))):
        pq = O.quantize_vectors(X[:, chans], P[64 * g:64 * (g + 1)][:, chans], bits)
        assert np.array_equal(mq["idx"][:, 64 * g:64 * (g + 1)], pq["idx"])
        np.testing.assert_allclose(mq["u"][:, 64 * g:64 * (g + 1)], pq["u"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(mq["n_O" if g == 0 else "n_R"], pq["n"], rtol=1e-15)


def test_pages_turbo3_bits_and_compression():
    """A 3.5-bit row (half at 4 bits, half at 3) packs 128 codes into 56 bytes; 16 / 3.5 = 4.57
    is the pages' 4.6x at their printed precision."""
    bits_per_value = (64 * BITS[0] + 64 * BITS[1]) / 128
    assert bits_per_value == GOLDEN["turbo3_bits_per_value"]["value"]
    idx = np.zeros((1, 128), dtype=np.int64)
    assert O.pack_codes_mixed(idx, *BITS, O.k_slot_of_coord_mixed).shape == (1, 56)
    assert round(16 / bits_per_value, GOLDEN["turbo3_compression_vs_fp16"]["printed_digits"]) == \
        GOLDEN["turbo3_compression_vs_fp16"]["value"]


def test_mixed_mse_is_the_average_of_the_pages_tq3_and_tq4():
    """Isotropic vectors: each half holds half the energy, so the normalized MSE is the mean of
    the 4-bit and 3-bit figures the pages print (0.009 and 0.034), within 5%."""
    rng = np.random.default_rng(11)
    X = rng.standard_normal((20000, 128))
    oc = np.arange(0, 128, 2)
    P = W.make_block_rotation(77, oc).astype(np.float64)
    q = O.quantize_vectors_mixed(X, P, oc, *BITS)
    xh = q["khat"] @ P  # back to the channel basis
    nmse = np.mean(np.sum((X - xh) ** 2, 1) / np.sum(X ** 2, 1))
    want = (GOLDEN["tq4_normalized_mse"]["value"] + GOLDEN["tq3_normalized_mse"]["value"]) / 2
    assert abs(nmse - want) <= 0.05 * want, nmse


def test_pack_roundtrip_and_hand_example():
    rng = np.random.default_rng(3)
    idx = np.concatenate([rng.integers(0, 16, (50, 64)), rng.integers(0, 8, (50, 64))], 1)
    for slot in (O.k_slot_of_coord_mixed, O.v_slot_of_coord_mixed):
        assert np.array_equal(O.unpack_codes_mixed(O.pack_codes_mixed(idx, *BITS, slot), *BITS, slot), idx)
    # key coordinate 64 + 19 = half R, j' = 19 = 16*1 + 8*0 + 2*1 + 1 -> slot 16*1 + 4*1 + 0 + 1 = 21:
    # 3-bit code 5 = 0b101 at bits 63..65 of the R stream, which starts at byte 32
    one = np.zeros((1, 128), dtype=np.int64)
    one[0, 64 + 19] = 5
    row = O.pack_codes_mixed(one, *BITS, O.k_slot_of_coord_mixed)[0]
    want = np.zeros(56, dtype=np.uint8)
    want[32 + 63 // 8] |= 1 << (63 % 8)   # bit 0 of the code
    want[32 + 65 // 8] |= 1 << (65 % 8)   # bit 2
    assert np.array_equal(row, want)


def test_zero_half():
    """A vector with all non-outlier channels 0: n_R = 0, u_R = 0 (codes at the middle cell) and
    the dequantized half R is the middle centroid times 0."""
    _, oc, P, X = _setup(n=4)
    rest = np.setdiff1d(np.arange(128), oc)
    X[:, rest] = 0
    q = O.quantize_vectors_mixed(X, P, oc, *BITS)
    assert np.all(q["n_R"] == 0) and np.all(q["u"][:, 64:] == 0)
    assert np.all(q["idx"][:, 64:] == 4) and np.all(q["khat"][:, 64:] == 0)


def test_decode_without_qjl_equals_exact_attention_on_dequantized_cache():
    """Brute force: softmax attention over khat, vhat mapped back to the channel basis."""
    w = W.CONFIGS["llama3_8b_32k"].scaled(T=37, B=1, Hkv=2, Hq=4)
    oc = W.outlier_channels_for(w)
    P = W.make_block_rotation(1000 + w.seed, oc)
    K = W.make_kv(w, "k").double().numpy()
    V = W.make_kv(w, "v").double().numpy()
    q = W.make_queries(w).double().numpy()
    c = O.quantize_cache_mixed(K, V, P, oc, BITS, BITS, None)
    got = O.decode_attention_mixed(q, P, None, c, BITS, BITS, 37)
    P64 = np.asarray(P, np.float64)
    for b in range(1):
        for h in range(4):
            kv = h // 2
            kh = O.dequantize_mixed(c["k_codes"][b, kv], c["k_norm"][b, kv], BITS, O.k_slot_of_coord_mixed) @ P64
            vh = O.dequantize_mixed(c["v_codes"][b, kv], c["v_norm"][b, kv], BITS, O.v_slot_of_coord_mixed) @ P64
            s = [sum(q[b, h, j] * kh[i, j] for j in range(128)) / math.sqrt(128) for i in range(37)]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            want = sum(e[i] * vh[i] for i in range(37)) / sum(e)
            np.testing.assert_allclose(got[b, h], want, rtol=0, atol=1e-10)


def test_qjl_estimator_unbiased_on_the_mixed_residual():
    """Over 10^4 sketch draws the QJL-corrected estimate of <q, k> is unbiased within 3 standard
    errors (the estimator of tproger.ru 'Step 2: QJL' with the block-rotated residual)."""
    rng = np.random.default_rng(21)
    oc = np.sort(rng.permutation(128)[:64])
    P = W.make_block_rotation(99, oc).astype(np.float64)
    k = rng.standard_normal(128) * np.exp(0.7 * rng.standard_normal(128))
    qv = rng.standard_normal(128)
    m = 128
    ests = []
    for t in range(10000):
        S = np.random.default_rng(1000 + t).standard_normal((m, 128))
        kq = O.quantize_vectors_mixed(k[None], P, oc, *BITS, S)
        qp = P @ qv
        est = kq["khat"][0] @ qp + kq["rnorm"][0] * math.sqrt(math.pi / 2) / m * ((2.0 * kq["signs"][0] - 1.0) @ (S @ qp))
        ests.append(est)
    ests = np.array(ests)
    se = ests.std(ddof=1) / math.sqrt(len(ests))
    assert abs(ests.mean() - qv @ k) < 3 * se, (ests.mean(), qv @ k, se)
    # dropping the correction leaves a bias many standard errors wide
    kq = O.quantize_vectors_mixed(k[None], P, oc, *BITS)
    assert abs(kq["khat"][0] @ (P @ qv) - qv @ k) > 10 * se
