"""Pins for the CPU oracle: closed forms, Lloyd conditions checked by independent
quadrature, the pages' printed figures, brute force on tiny inputs, invariants and
QJL unbiasedness.  Each test is chosen so that a plausible slip in the oracle (a
dropped term, a wrong sign or index, a transposed operand, a wrong bit position)
fails at least one of them.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy import integrate

import workloads as W
from oracle import tq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")


def pages():
    with open(GOLDEN) as f:
        return json.load(f)


def phi(x):
    return math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)


# --------------------------------------------------------------------------- codebook

def test_one_bit_closed_form():
    """b = 1: the Lloyd-Max quantizer of N(0,1) is +-sqrt(2/pi) with distortion 1 - 2/pi."""
    c, t, dist, _ = O.lloyd_max_gaussian(1)
    assert np.allclose(c, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], atol=1e-13, rtol=0)
    assert t[0] == 0.0
    assert abs(dist - (1 - 2 / math.pi)) < 1e-13


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_centroid_condition_by_quadrature(bits):
    """Each centroid is the conditional mean of its cell, by independent numerical quadrature."""
    c, t, _, _ = O.lloyd_max_gaussian(bits)
    edges = [-np.inf] + list(t) + [np.inf]
    for k in range(len(c)):
        a, b = edges[k], edges[k + 1]
        mass = integrate.quad(phi, a, b, epsabs=1e-14, epsrel=1e-13)[0]
        mom = integrate.quad(lambda x: x * phi(x), a, b, epsabs=1e-14, epsrel=1e-13)[0]
        assert abs(mom / mass - c[k]) < 1e-10, (bits, k)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_midpoint_condition_and_symmetry(bits):
    c, t, _, _ = O.lloyd_max_gaussian(bits)
    assert np.all(np.diff(c) > 0)
    assert np.array_equal(c, -c[::-1])
    assert np.array_equal(t, 0.5 * (c[:-1] + c[1:]))


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_distortion_by_quadrature(bits):
    """Reported distortion equals E[(X - Q(X))^2] integrated cell by cell."""
    c, t, dist, _ = O.lloyd_max_gaussian(bits)
    edges = [-np.inf] + list(t) + [np.inf]
    total = 0.0
    for k in range(len(c)):
        total += integrate.quad(lambda x: (x - c[k]) ** 2 * phi(x), edges[k], edges[k + 1],
                                epsabs=1e-14, epsrel=1e-12)[0]
    assert abs(total - dist) < 1e-10


def test_distortion_decreasing_and_within_pages_factor():
    """D_b strictly decreases in b, and 4^-b <= D_b <= 2.7 * 4^-b (the pages' near-optimality
    factor against the Gaussian distortion-rate bound 4^-b)."""
    factor = pages()["near_optimality_factor"]["value"]
    ds = [O.lloyd_max_gaussian(b)[2] for b in range(1, 5)]
    assert all(ds[i] > ds[i + 1] for i in range(3))
    for b, d in zip(range(1, 5), ds):
        assert 4.0 ** -b <= d <= factor * 4.0 ** -b, (b, d)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_stored_codebook(bits):
    cb = O.codebook(bits)
    c16 = cb.centroids
    assert np.array_equal(c16.astype(np.float16).astype(np.float64), c16)
    assert np.all(np.abs(c16 - cb.lloyd_centroids) <= 2.0 ** -11 * np.abs(cb.lloyd_centroids))
    assert np.array_equal(c16, -c16[::-1])
    assert np.all(np.diff(cb.thresholds) > 0)
    assert np.array_equal(cb.thresholds.astype(np.float32).astype(np.float64), cb.thresholds)
    assert cb.thresholds[len(cb.thresholds) // 2] == 0.0


def test_index_tie_goes_up():
    t = O.codebook(2).thresholds
    u = np.array([t[0], np.nextafter(t[0], -np.inf), 0.0, -0.0, t[2], 100.0, -100.0])
    assert O.quantize_index(u, t).tolist() == [1, 0, 2, 2, 3, 3, 0]


# --------------------------------------------------------------------------- rotation / sketch

@pytest.mark.parametrize("seed", [1000, 1001, 1002, 1003, 1004])
def test_rotation_orthogonal(seed):
    Pi = W.make_rotation(seed).astype(np.float64)
    assert np.max(np.abs(Pi @ Pi.T - np.eye(128))) <= 1e-6
    assert np.max(np.abs(Pi.T @ Pi - np.eye(128))) <= 1e-6


def test_sketch_is_fp16_gaussian():
    S = W.make_qjl_matrix(2001)
    assert np.array_equal(S.astype(np.float16).astype(np.float32), S)
    assert abs(S.mean()) < 0.03 and abs(S.std() - 1.0) < 0.02


# --------------------------------------------------------------------------- pages' figures

def _normalized_mse(X, Pi, bits):
    r = O.quantize_vectors(X, Pi, bits)
    xh = (r["n"][:, None] / math.sqrt(128)) * O.codebook(bits).centroids[r["idx"]] @ Pi.astype(
        np.float64)
    return float(np.mean(np.sum((X - xh) ** 2, 1) / np.sum(X ** 2, 1)))


def test_pages_normalized_mse_isotropic():
    """Random-direction vectors reproduce TQ3 MSE 0.034 and TQ4 MSE 0.009 at the printed precision."""
    p = pages()
    g = torch.Generator().manual_seed(7)
    X = torch.randn(40000, 128, generator=g, dtype=torch.float64).numpy()
    Pi = W.make_rotation(1007)
    for bits, key in ((3, "tq3_normalized_mse"), (4, "tq4_normalized_mse")):
        mse = _normalized_mse(X, Pi, bits)
        half_unit = 0.5 * 10.0 ** -p[key]["printed_digits"]
        assert abs(mse - p[key]["value"]) <= half_unit, (bits, mse)


def test_pages_normalized_mse_single_head_keys():
    """Keys of the single-head workload (fp32, 4 outlier channels x20) also match 0.034 / 0.009."""
    p = pages()
    w = W.CONFIGS["single_head_4k"]
    X = W.make_kv(w, "k").reshape(-1, 128).double().numpy()
    Pi = W.rotation_for(w)
    for bits, key in ((3, "tq3_normalized_mse"), (4, "tq4_normalized_mse")):
        mse = _normalized_mse(X, Pi, bits)
        assert abs(mse - p[key]["value"]) <= 0.5 * 10.0 ** -p[key]["printed_digits"], (bits, mse)


def test_pages_block_bytes_and_compression():
    """A 3-bit value row is 48 code bytes + a 4-byte norm = 52 B per 128 values; 128 fp16 values
    take 256 B, so TQ3 compresses 4.9x and TQ4 (64 + 4 B) 3.8x at the printed precision."""
    p = pages()
    idx = np.zeros((1, 128), dtype=np.int64)
    assert O.pack_codes(idx, 3, O.v_slot_of_coord).shape[1] + 4 == p["tq3_block_bytes_per_128"]["value"]
    w3 = W.CONFIGS["llama3_8b_32k"]
    assert w3.v_row_bytes() == p["tq3_block_bytes_per_128"]["value"]
    w4 = W.CONFIGS["llama3_8b_128k_b4"]
    assert round(256 / w3.v_row_bytes(), 1) == p["tq3_compression_vs_fp16"]["value"]
    assert round(256 / w4.v_row_bytes(), 1) == p["tq4_compression_vs_fp16"]["value"]


# --------------------------------------------------------------------------- packing layout

def test_pack_hand_example_keys():
    """Pi = I, x = e_2, 3 bits: u_2 = sqrt(128) -> code 7, every other u_j = 0 -> code 4 (tie at
    the middle threshold 0 goes up).  Coordinate 2 = 16*0 + 8*0 + 2*1 + 0 sits at slot 32.
    Row bits set: 3s+2 for every slot s (code 4 = 0b100) plus bits 96, 97 (slot 32 = 0b111)."""
    x = np.zeros((1, 128))
    x[0, 2] = 1.0
    r = O.quantize_vectors(x, np.eye(128), 3)
    assert r["idx"][0, 2] == 7 and np.all(np.delete(r["idx"][0], 2) == 4)
    row = O.pack_codes(r["idx"], 3, O.k_slot_of_coord)[0]
    expect = bytearray(48)
    for s in range(128):
        k = 3 * s + 2
        expect[k // 8] |= 1 << (k % 8)
    for k in (96, 97):
        expect[k // 8] |= 1 << (k % 8)
    assert bytes(row) == bytes(expect)
    assert row[0] == 0x24 and row[1] == 0x49 and row[2] == 0x92
    assert row[12] == 0x27  # bits 96..103: 96, 97, 98, 101


def test_pack_hand_example_values_and_signs():
    """Value rows: coordinate 9 = 8*1 + 1 sits at slot 16*1 + 1 = 17.  Sign rows: sketch row
    3 = 2*1 + 1 (tau = 1, eps = 1) sits at bit 32*1 + 0 + 16 = 48."""
    idx = np.zeros((1, 128), dtype=np.int64)
    idx[0, 9] = 1
    row = O.pack_codes(idx, 2, O.v_slot_of_coord)[0]
    assert np.flatnonzero(row).tolist() == [34 // 8] and row[4] == 1 << (34 % 8)
    s = np.zeros((1, 128), dtype=np.int64)
    s[0, 3] = 1
    srow = O.pack_signs(s)[0]
    assert np.flatnonzero(srow).tolist() == [6] and srow[6] == 1
    # the three slot maps are permutations of 0..127
    for f in (O.k_slot_of_coord, O.v_slot_of_coord, O.sign_bit_of_row):
        assert sorted(f(j) for j in range(128)) == list(range(128))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    idx = rng.integers(0, 1 << bits, size=(17, 128))
    for f in (O.k_slot_of_coord, O.v_slot_of_coord):
        assert np.array_equal(O.unpack_codes(O.pack_codes(idx, bits, f), bits, f), idx)
    s = rng.integers(0, 2, size=(17, 128))
    assert np.array_equal(O.unpack_signs(O.pack_signs(s)), s)


# --------------------------------------------------------------------------- quantize special cases

def test_zero_vector():
    r = O.quantize_vectors(np.zeros((1, 128)), W.make_rotation(1000), 3, W.make_qjl_matrix(2000))
    assert r["n"][0] == 0 and np.all(r["u"] == 0) and np.all(r["idx"] == 4)
    assert r["rnorm"][0] == 0.0


def test_quantize_scale_invariance():
    """Codes depend only on the direction of x; norms scale with it."""
    w = W.CONFIGS["llama3_8b_32k"].scaled(T=16, B=1, Hkv=1, Hq=4)
    X = W.make_kv(w, "k").reshape(-1, 128).double().numpy()
    Pi, S = W.rotation_for(w), W.qjl_for(w)
    a = O.quantize_vectors(X, Pi, 3, S)
    b = O.quantize_vectors(4.0 * X, Pi, 3, S)
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["signs"], b["signs"])
    assert np.allclose(4.0 * a["n"], b["n"]) and np.allclose(4.0 * a["rnorm"], b["rnorm"])


def test_rotation_is_applied_as_pi_times_x():
    """A transposed rotation would give different codes: pin the orientation with a vector
    equal to a row of Pi (then u = sqrt(d) e_row)."""
    Pi = W.make_rotation(1003)
    x = Pi[5:6].astype(np.float64)
    r = O.quantize_vectors(x, Pi, 4)
    assert r["idx"][0, 5] == 15
    assert abs(r["u"][0, 5] - math.sqrt(128)) < 1e-5


# --------------------------------------------------------------------------- attention

def _loop_attention(q, K, V, scale):
    s = [scale * sum(q[j] * K[i][j] for j in range(len(q))) for i in range(len(K))]
    m = max(s)
    w = [math.exp(x - m) for x in s]
    tot = sum(w)
    return [sum(w[i] * V[i][j] for i in range(len(K))) / tot for j in range(len(V[0]))]


@pytest.mark.parametrize("T", [1, 7, 64])
def test_exact_attention_brute_force(T):
    rng = np.random.default_rng(T)
    q = rng.standard_normal((1, 2, 8))
    K = rng.standard_normal((1, 1, T, 8)) * 2
    V = rng.standard_normal((1, 1, T, 8))
    out = O.exact_attention(q, K, V, scale=0.7)
    for h in range(2):
        ref = _loop_attention(q[0, h].tolist(), K[0, 0].tolist(), V[0, 0].tolist(), 0.7)
        assert np.allclose(out[0, h], ref, atol=1e-13, rtol=0)


def _dequant(cache, bits_k, bits_v, Pi):
    d = 128
    Pi64 = Pi.astype(np.float64)
    B, H, T, _ = cache["k_codes"].shape
    kidx = O.unpack_codes(cache["k_codes"].reshape(-1, 16 * bits_k), bits_k, O.k_slot_of_coord)
    vidx = O.unpack_codes(cache["v_codes"].reshape(-1, 16 * bits_v), bits_v, O.v_slot_of_coord)
    kh = (cache["k_norm"].reshape(-1, 1).astype(np.float64) / math.sqrt(d)) * O.codebook(bits_k).centroids[kidx]
    vh = (cache["v_norm"].reshape(-1, 1).astype(np.float64) / math.sqrt(d)) * O.codebook(bits_v).centroids[vidx]
    return (kh @ Pi64).reshape(B, H, T, d), (vh @ Pi64).reshape(B, H, T, d)


def test_decode_without_qjl_equals_exact_attention_on_dequantized_cache():
    """With QJL off, decode over the packed cache is exact softmax attention over the
    dequantized keys/values Pi^T (n/sqrt(d)) c[idx], with GQA and a ragged seq_len."""
    w = W.CONFIGS["llama3_8b_32k"].scaled(T=40, B=2, Hkv=2, Hq=6)
    K = W.make_kv(w, "k").double().numpy()
    V = W.make_kv(w, "v").double().numpy()
    q = W.make_queries(w).double().numpy()
    Pi = W.rotation_for(w)
    cache = O.quantize_cache(K, V, Pi, 3, 2, None)
    Kh, Vh = _dequant(cache, 3, 2, Pi)
    for seq_len in (40, 33, 1):
        got = O.decode_attention(q, Pi, None, cache, 3, 2, seq_len)
        ref = O.exact_attention(q, Kh[:, :, :seq_len], Vh[:, :, :seq_len])
        assert np.allclose(got, ref, atol=1e-11, rtol=0)
    assert np.all(O.decode_attention(q, Pi, None, cache, 3, 2, 0) == 0)


def test_attention_error_decreases_with_bits():
    w = W.CONFIGS["llama3_8b_32k"].scaled(T=256, B=1, Hkv=2, Hq=8)
    K = W.make_kv(w, "k").double().numpy()
    V = W.make_kv(w, "v").double().numpy()
    q = W.make_queries(w).double().numpy()
    Pi = W.rotation_for(w)
    ref = O.exact_attention(q, K, V)
    errs = []
    for b in (2, 3, 4):
        cache = O.quantize_cache(K, V, Pi, b, b, None)
        errs.append(np.linalg.norm(O.decode_attention(q, Pi, None, cache, b, b, 256) - ref))
    assert errs[0] > errs[1] > errs[2]


def test_qjl_estimator_unbiased_and_variance():
    """Over 10^4 sketch seeds (fixed q, k, Pi) the QJL-corrected score is unbiased for <q,k>
    within 3 standard errors, and its variance matches the closed form
    (pi/(2m)) ||r||^2 ||q||^2 - <q,r>^2 / m  (from E[(s.q) sign(s.r)] = sqrt(2/pi) <q,r>/||r||)."""
    w = W.CONFIGS["llama3_8b_32k"].scaled(T=1, B=1, Hkv=1, Hq=1)
    k = W.make_kv(w, "k").double().numpy().reshape(1, 128)
    q = W.make_queries(w).double().numpy().reshape(128)
    Pi = W.rotation_for(w)
    base = O.quantize_vectors(k, Pi, 3)
    codes = O.pack_codes(base["idx"], 3, O.k_slot_of_coord)
    kn = base["n"].astype(np.float32)
    # residual in original units: r = Pi^T (n / sqrt(d)) rho
    r = (Pi.astype(np.float64).T @ (base["n"][0] / math.sqrt(128) * base["rho"][0]))
    k_mse = k[0] - r
    # tilt q toward the residual so that dropping the correction is a large, visible bias
    q = q + 2.0 * np.linalg.norm(q) * r / np.linalg.norm(r)
    ests = []
    for seed in range(10000):
        S = W.make_qjl_matrix(50000 + seed)
        qv = O.quantize_vectors(k, Pi, 3, S)
        ests.append(O.score_estimates(q, Pi, S, codes, kn, 3, O.pack_signs(qv["signs"]),
                                      qv["rnorm"].astype(np.float32))[0])
    ests = np.array(ests)
    truth = float(q @ k[0])
    mse_part = float(q @ k_mse)
    se = ests.std(ddof=1) / math.sqrt(len(ests))
    assert abs(ests.mean() - truth) < 3 * se, (ests.mean(), truth, se)
    # the uncorrected estimate is biased by <q, r>, far outside the same band
    assert abs(mse_part - truth) > 10 * se
    m = 128
    rn2 = float(r @ r)
    var_closed = math.pi / (2 * m) * rn2 * float(q @ q) - float(q @ r) ** 2 / m
    assert abs(ests.var(ddof=1) / var_closed - 1.0) < 0.06, (ests.var(ddof=1), var_closed)


def test_exemption_masks():
    t = O.codebook(2).thresholds
    u = np.array([[t[0] + 5e-7, t[0] + 2e-6, 0.0, 1.0]])
    m = O.code_exempt(u, 2)
    assert m.tolist() == [[True, False, True, False]]
    sp = np.array([[1e-6, 1e-4, -1e-6, 0.5]])
    assert O.sign_exempt(sp, np.zeros((1, 4), bool)).tolist() == [[True, False, True, False]]
    assert O.sign_exempt(sp, m).all()
