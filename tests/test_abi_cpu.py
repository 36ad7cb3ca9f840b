"""C-ABI checks that need no GPU: the library loads, exports every function include/tq.h
declares, builds the same codebook as the oracle, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import numpy as np
import pytest

import decode_attention_11_b200 as tq
from oracle import tq_oracle as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "tq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert set(names) == set(tq.EXPORTED)
    L = tq.lib()
    for n in names:
        assert hasattr(L, n), n
    assert tq.version() >= 100


def test_debug_library_exports_the_same_functions():
    """libtq_b200_debug.so (decode bounds checks, built by build(debug=True)) loads and exports
    every declared function too, so TQ_DEBUG=1 can stand in for the release library."""
    from decode_attention_11_b200.build import DEBUG_LIB
    if not os.path.exists(DEBUG_LIB):
        pytest.skip("debug library not built (python -m decode_attention_11_b200.build --debug)")
    L = ctypes.CDLL(DEBUG_LIB)
    for n in declared_functions():
        assert hasattr(L, n), n
    L.tq_version.restype = ctypes.c_int
    assert L.tq_version() == tq.version()


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_matches_oracle_bit_exact(bits):
    c, t, dist = tq.build_codebook(bits)
    cb = O.codebook(bits)
    assert np.array_equal(c.astype(np.float64), cb.centroids)
    assert np.array_equal(t.astype(np.float64), cb.thresholds)
    assert abs(dist - cb.lloyd_distortion) < 1e-12


def test_codebook_errors():
    with pytest.raises(tq.TqError) as e:
        tq.build_codebook(0)
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    with pytest.raises(tq.TqError) as e:
        tq.build_codebook(4, max_iter=3)
    assert e.value.status == tq.TQ_ERR_NO_CONVERGENCE
    assert "iterations" in tq.last_error()
    assert tq.status_string(tq.TQ_ERR_WORKSPACE).startswith("TQ_ERR_WORKSPACE")
    assert tq.status_string(99) == "unknown tq_status"


FAKE = 0x10000  # aligned, never dereferenced: validation fails or returns before any device work


def fake_cache(**kw):
    c = dict(B=1, Hkv=2, T_cap=64, head_dim=128, k_bits=3, v_bits=3, qjl_m=128,
             k_codes=FAKE, k_signs=FAKE, k_norm=FAKE, k_rnorm=FAKE, v_codes=FAKE, v_norm=FAKE)
    c.update(kw)
    return tq._Cache(**c)


def fake_params(**kw):
    p = dict(Pi=FAKE, S=FAKE, k_centroids=FAKE, k_thresholds=FAKE, v_centroids=FAKE, v_thresholds=FAKE)
    p.update(kw)
    return tq._Params(**p)


def quantize_status(params=None, cache=None, k=FAKE, v=FAKE, dtype=tq.TQ_BF16, strides=(16384, 8192, 128),
                    T_new=8, t_offset=0):
    L = tq.lib()
    return L.tq_quantize(ctypes.byref(params or fake_params()), k, v, dtype, *strides, T_new, t_offset,
                         ctypes.byref(cache or fake_cache()), None)


def test_quantize_argument_errors():
    assert quantize_status(cache=fake_cache(head_dim=64)) == tq.TQ_ERR_UNSUPPORTED
    assert quantize_status(cache=fake_cache(k_bits=5)) == tq.TQ_ERR_UNSUPPORTED
    assert quantize_status(cache=fake_cache(qjl_m=64)) == tq.TQ_ERR_UNSUPPORTED
    assert quantize_status(cache=fake_cache(k_codes=None)) == tq.TQ_ERR_INVALID_ARG
    assert quantize_status(cache=fake_cache(k_norm=FAKE + 4)) == tq.TQ_ERR_INVALID_ARG
    assert quantize_status(cache=fake_cache(k_signs=None)) == tq.TQ_ERR_INVALID_ARG
    assert quantize_status(params=fake_params(S=None)) == tq.TQ_ERR_INVALID_ARG
    assert quantize_status(dtype=7) == tq.TQ_ERR_UNSUPPORTED
    assert quantize_status(T_new=60, t_offset=10) == tq.TQ_ERR_INVALID_ARG
    assert quantize_status(T_new=-1) == tq.TQ_ERR_INVALID_ARG
    assert quantize_status(k=None) == tq.TQ_ERR_INVALID_ARG
    assert quantize_status(k=FAKE + 2) == tq.TQ_ERR_INVALID_ARG
    assert quantize_status(strides=(16384, 8192, 100)) == tq.TQ_ERR_INVALID_ARG
    assert "stride" in tq.last_error()
    # T_new = 0 enqueues nothing and succeeds without a device
    assert quantize_status(T_new=0) == tq.TQ_OK
    # QJL off: sign arrays and S may be NULL
    assert quantize_status(cache=fake_cache(qjl_m=0, k_signs=None, k_rnorm=None),
                           params=fake_params(S=None), T_new=0) == tq.TQ_OK


def decode_status(cache=None, params=None, q=FAKE, Hq=8, seq_len=64, out=FAKE, ws=FAKE, ws_bytes=1 << 30):
    L = tq.lib()
    return L.tq_decode_attn(ctypes.byref(params or fake_params()), q, tq.TQ_F32, Hq,
                            ctypes.byref(cache or fake_cache()), seq_len, 0.0, out, ws, ws_bytes, None)


def test_decode_argument_errors():
    assert decode_status(Hq=7) == tq.TQ_ERR_INVALID_ARG
    assert decode_status(seq_len=65) == tq.TQ_ERR_INVALID_ARG
    assert decode_status(seq_len=-1) == tq.TQ_ERR_INVALID_ARG
    assert decode_status(out=None) == tq.TQ_ERR_INVALID_ARG
    assert decode_status(q=FAKE + 8) == tq.TQ_ERR_INVALID_ARG
    assert decode_status(cache=fake_cache(v_bits=1)) == tq.TQ_ERR_UNSUPPORTED
    assert decode_status(ws_bytes=16) == tq.TQ_ERR_WORKSPACE
    assert "need" in tq.last_error()


def test_workspace_size():
    c = fake_cache()
    L = tq.lib()
    n = L.tq_decode_workspace_size(1, 8, ctypes.byref(c), 64)
    assert n >= 4 * 8 * 132  # at least one (max, sum, pad, pad, o[128]) partial per query head
    assert L.tq_decode_workspace_size(1, 7, ctypes.byref(c), 64) == 0
    assert L.tq_decode_workspace_size(1, 8, None, 64) == 0
    big = L.tq_decode_workspace_size(4, 32, ctypes.byref(fake_cache(B=4, Hkv=8, T_cap=131072)), 131072)
    assert big < 64 << 20


def step_status(cache=None, params=None, k=FAKE, v=FAKE, kv_dtype=tq.TQ_BF16, q=FAKE, Hq=8, t=10,
                out=FAKE, ws=FAKE, ws_bytes=1 << 30):
    L = tq.lib()
    return L.tq_decode_step(ctypes.byref(params or fake_params()), k, v, kv_dtype, q, tq.TQ_F32, Hq,
                            ctypes.byref(cache or fake_cache()), t, 0.0, out, ws, ws_bytes, None)


def test_decode_step_argument_errors():
    """Every argument of tq_decode_step is checked before anything is enqueued."""
    assert step_status(t=64) == tq.TQ_ERR_INVALID_ARG  # T_cap = 64: the new row must exist
    assert step_status(t=-1) == tq.TQ_ERR_INVALID_ARG
    assert step_status(Hq=7) == tq.TQ_ERR_INVALID_ARG
    assert step_status(out=None) == tq.TQ_ERR_INVALID_ARG
    assert step_status(q=FAKE + 8) == tq.TQ_ERR_INVALID_ARG
    assert step_status(ws_bytes=16) == tq.TQ_ERR_WORKSPACE
    assert "need" in tq.last_error()
    assert step_status(kv_dtype=7) == tq.TQ_ERR_UNSUPPORTED
    assert step_status(k=None) == tq.TQ_ERR_INVALID_ARG
    assert step_status(v=FAKE + 4) == tq.TQ_ERR_INVALID_ARG
    assert step_status(cache=fake_cache(k_bits=5)) == tq.TQ_ERR_UNSUPPORTED
    assert step_status(params=fake_params(S_Pi=FAKE + 8)) == tq.TQ_ERR_INVALID_ARG


def test_sketch_rotation_and_hadamard_builder_argument_errors():
    L = tq.lib()
    assert L.tq_sketch_rotation(None, FAKE, 128, FAKE, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_sketch_rotation(FAKE, FAKE + 4, 128, FAKE, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_sketch_rotation(FAKE, FAKE, 0, FAKE, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_build_hadamard_rotation(1, None) == tq.TQ_ERR_INVALID_ARG
    assert quantize_status(params=fake_params(S_Pi=FAKE + 8)) == tq.TQ_ERR_INVALID_ARG


def test_debug_quantize_stall_argument_check():
    """The failure-handling test hook refuses a non-positive wait limit (no device needed)."""
    L = tq.lib()
    assert L.tq_debug_quantize_stall(1, 0) == tq.TQ_ERR_INVALID_ARG
    assert "wait_cycles" in tq.last_error()
    assert L.tq_debug_quantize_stall(0, 0) == tq.TQ_OK


def test_decode_step_fused_choice():
    """Where the decode step runs as one fused launch (host logic, the 148-SM plan without a GPU):
    long contexts yes; many short units (a CTA's range crossing several units) and the mixed
    layout no; invalid sizes -1."""
    L = tq.lib()
    long_ctx = fake_cache(B=1, Hkv=8, T_cap=32768)
    assert L.tq_decode_step_fused(ctypes.byref(long_ctx), 32, 32767) == 1
    assert L.tq_decode_step_fused(ctypes.byref(long_ctx), 32, 4000) == 1
    short = fake_cache(B=8, Hkv=8, T_cap=64)
    assert L.tq_decode_step_fused(ctypes.byref(short), 32, 10) == 0
    mixed = fake_cache(B=1, Hkv=8, T_cap=32768, k_bits=4, v_bits=4, layout=tq.TQ_LAYOUT_MIXED)
    assert L.tq_decode_step_fused(ctypes.byref(mixed), 32, 32767) == 0
    assert L.tq_decode_step_fused(ctypes.byref(long_ctx), 30, 100) == -1
    assert L.tq_decode_step_fused(ctypes.byref(long_ctx), 32, 32768) == -1
