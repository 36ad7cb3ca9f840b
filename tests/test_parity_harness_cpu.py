"""CPU checks of the GPU parity harness itself (tests/_parity.py): a cache written by the oracle
passes, and each kind of planted mistake (a code, a sign, a norm, ||r||) in a clean row is caught,
while a different code at an exempt coordinate is tolerated and counted."""
import types

import numpy as np
import pytest
import torch

import workloads as W
from oracle import tq_oracle as O

from _parity import compare_quantized, exemption_free_inputs

KEYS = ["k_codes", "k_signs", "k_norm", "k_rnorm", "v_codes", "v_norm"]


def _workload():
    return W.CONFIGS["llama3_8b_128k_b4"].scaled(T=40, B=1, Hkv=2, Hq=8)


def _inputs_with_exempt_coordinate(w):
    """Seeded recipe inputs, with key row (0, 1, 7) replaced by a vector whose rotated coordinate
    5 equals a threshold (x = Pi^T u for such a u), so that coordinate is exempt."""
    K = W.make_kv(w, "k").double().numpy()
    V = W.make_kv(w, "v").double().numpy()
    Pi = W.rotation_for(w).astype(np.float64)
    u = np.random.default_rng(5).standard_normal(128)
    t = O.codebook(w.k_bits).thresholds[9]
    u[5] = 0.0
    u *= np.sqrt(128.0 - t * t) / np.linalg.norm(u)  # ||u|| = sqrt(128): u = sqrt(d) Pi x / ||x||
    u[5] = t
    K[0, 1, 7] = Pi.T @ u
    return K, V


def _fake_cache(w, K, V):
    c = O.quantize_cache(K, V, W.rotation_for(w), w.k_bits, w.v_bits, W.qjl_for(w))
    return types.SimpleNamespace(**{k: torch.as_tensor(np.ascontiguousarray(c[k])) for k in KEYS}), c


def test_oracle_cache_passes_and_counts_the_exempt_coordinate():
    w = _workload()
    K, V = _inputs_with_exempt_coordinate(w)
    cache, _ = _fake_cache(w, K, V)
    st = compare_quantized(w, cache, K, V, 0)
    assert st["vectors"] == w.B * w.Hkv * w.T
    assert st["exempt_codes"] >= 1 and st["code_mismatch_in_band"] == 0


def test_other_code_at_an_exempt_coordinate_is_tolerated():
    w = _workload()
    K, V = _inputs_with_exempt_coordinate(w)
    cache, c = _fake_cache(w, K, V)
    idx = c["k_idx"][0, 1, 7].copy()
    idx[5] -= 1  # the other side of the threshold
    cache.k_codes[0, 1, 7] = torch.as_tensor(O.pack_codes(idx[None], w.k_bits, O.k_slot_of_coord)[0])
    st = compare_quantized(w, cache, K, V, 0)
    assert st["code_mismatch_in_band"] == 1


@pytest.mark.parametrize("what", ["k_code", "v_code", "sign", "k_norm", "v_norm", "rnorm", "offset"])
def test_planted_mistake_in_a_clean_row_is_caught(what):
    w = _workload()
    K, V = _inputs_with_exempt_coordinate(w)
    cache, _ = _fake_cache(w, K, V)
    b, h, t = 0, 0, 11
    if what == "k_code":
        cache.k_codes[b, h, t, 3] ^= 0x10
    elif what == "v_code":
        cache.v_codes[b, h, t, 0] ^= 0x01
    elif what == "sign":
        cache.k_signs[b, h, t, 15] ^= 0x80
    elif what == "k_norm":
        cache.k_norm[b, h, t] = cache.k_norm[b, h, t] * (1 + 2e-6)
    elif what == "v_norm":
        cache.v_norm[b, h, t] = cache.v_norm[b, h, t] * (1 - 2e-6)
    elif what == "rnorm":
        cache.k_rnorm[b, h, t] = cache.k_rnorm[b, h, t] * (1 + 3e-5)
    with pytest.raises(AssertionError):
        # "offset": the right cache compared as if written one row later
        compare_quantized(w, cache, K, V, 0 if what != "offset" else 1) if what != "offset" else \
            compare_quantized(w, cache, K[:, :, :-1], V[:, :, :-1], 1)


def test_exemption_free_inputs_have_no_exempt_case():
    w = W.CONFIGS["llama3_8b_32k"].scaled(T=300, B=1, Hkv=2, Hq=8)
    K, V = exemption_free_inputs(w)
    assert K.shape == (w.B, w.Hkv, w.T, 128) and K.dtype == torch.bfloat16
    Pi, S = W.rotation_for(w), W.qjl_for(w)
    kq = O.quantize_vectors(K.double().numpy().reshape(-1, 128), Pi, w.k_bits, S)
    vq = O.quantize_vectors(V.double().numpy().reshape(-1, 128), Pi, w.v_bits, None)
    assert not O.code_exempt(kq["u"], w.k_bits).any()
    assert not O.code_exempt(vq["u"], w.v_bits).any()
    assert not (np.abs(kq["sproj"]) <= O.SIGN_BAND).any()
    # the kept vectors are the recipe's own draws, in order
    big = W.make_kv(w.scaled(T=w.T + 64), "k")
    assert torch.equal(K[0, 0, 0], big[0, 0, 0]) or torch.equal(K[0, 0, 0], big[0, 0, 1])
