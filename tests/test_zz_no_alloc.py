"""Allocation-free decode entry point (tq_decode_attn_static), for callers that cannot allocate
device memory when they run decode (inside an allocator callback, under a runtime with a fixed
device footprint, in a plug-in host).  Its scratch is a fixed device array in the library.

Checked through the C ABI against tq_decode_attn (caller-provided workspace) on two calls in a
row, so the second call runs on scratch left over from the first.  Kept in a file of its own that
pytest collects last."""
import ctypes

import numpy as np
import pytest
import torch

import decode_attention_11_b200 as tq
import workloads as W

from _parity import ATTN_MAX_ABS, ATTN_REL_L2, attention_errors

pytestmark = pytest.mark.gpu


def _setup(name, **resize):
    w = W.CONFIGS[name].scaled(**resize)
    params = tq.Params.create(W.rotation_for(w), W.qjl_for(w), w.k_bits, w.v_bits)
    K = W.make_kv(w, "k", device="cuda")
    V = W.make_kv(w, "v", device="cuda")
    cache = tq.Cache.allocate(w.B, w.Hkv, w.T, w.k_bits, w.v_bits, w.qjl_m)
    tq.quantize(params, K, V, cache)
    q = W.make_queries(w, device="cuda")
    return w, params, cache, q


def _call_static(params, q, cache, seq_len, out):
    """tq_decode_attn_static through ctypes, returning the status code."""
    c = cache.as_c()
    p = params.as_c()
    return tq.lib().tq_decode_attn_static(ctypes.byref(p), q.data_ptr(), tq.TQ_F32, q.shape[1],
                                          ctypes.byref(c), int(seq_len), 0.0, out.data_ptr(), None)


def test_static_decode_matches_workspace_decode_two_calls():
    runs = [_setup("llama3_8b_128k_b4", T=6000, B=2, Hkv=2, Hq=8),
            _setup("llama3_70b_16k_b16", T=3000, B=3, Hkv=2, Hq=16)]
    for (w, params, cache, q), seq_len in zip(runs, (5999, 2048)):
        out_static = torch.full((w.B, w.Hq, 128), float("nan"), device="cuda")
        assert _call_static(params, q, cache, seq_len, out_static) == tq.TQ_OK, tq.last_error()
        ref = tq.decode_attn(params, q, cache, seq_len)
        torch.cuda.synchronize()
        got = out_static.cpu().numpy()
        exp = ref.cpu().numpy()
        assert np.isfinite(got).all()
        max_abs, rel = attention_errors(got, exp)
        assert max_abs <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, (max_abs, rel)
        # Both entry points run the same kernels with the same plan, so the results are the same
        # bits: a wrong scratch offset or a stale scratch read would show up here.
        assert torch.equal(out_static, ref)


def test_static_decode_rejects_sizes_above_the_limit():
    limit = tq.decode_static_workspace_limit()
    assert limit == 16 << 20
    w, params, cache, q = _setup("llama3_8b_32k", T=256, B=1, Hkv=8, Hq=32)
    # a cache description whose split-K scratch exceeds the limit (never dereferenced)
    big = cache.as_c()
    big.B, big.Hkv, big.T_cap = 64, 8, 1 << 20
    qbig = torch.empty(1, dtype=torch.float32, device="cuda")
    p = params.as_c()
    st = tq.lib().tq_decode_attn_static(ctypes.byref(p), qbig.data_ptr(), tq.TQ_F32, 64,
                                        ctypes.byref(big), 1 << 20, 0.0, qbig.data_ptr(), None)
    assert st == tq.TQ_ERR_WORKSPACE
    assert "static workspace" in tq.last_error()
