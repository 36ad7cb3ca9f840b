"""Failure handling of tq_quantize on the GPU without a fault: the test hook makes every CTA skip
its first tile load and shortens every wait, so the pipeline's bounded waits run out.  The kernel
must return promptly, record bit 0 in tq_quantize_device_errors and leave the context usable: the
next normal call on the same stream produces a correct cache.  Collected late (it sets, then
clears, the sticky error bits)."""
import time

import pytest
import torch

import decode_attention_11_b200 as tq
import workloads as W

from _parity import compare_quantized, gpu_inputs, params_for

pytestmark = pytest.mark.gpu


def test_quantize_wait_runs_out_reports_and_recovers():
    w = W.CONFIGS["llama3_8b_32k"].scaled(T=1000, B=1, Hkv=2, Hq=8)
    params = params_for(w)
    K, V, Kh, Vh = gpu_inputs(w)
    tq.reset_device_errors()
    assert tq.quantize_device_errors() == 0
    stalled = tq.Cache.allocate(w.B, w.Hkv, w.T, w.k_bits, w.v_bits, w.qjl_m)
    torch.cuda.synchronize()
    tq.debug_quantize_stall(True, 200_000)  # about 0.1 ms per wait at 2 GHz
    try:
        t0 = time.perf_counter()
        tq.quantize(params, K, V, stalled)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        tq.debug_quantize_stall(False)
    err = tq.quantize_device_errors()
    assert err & 1, err
    assert elapsed < 5.0, elapsed
    # the context is usable and the next call is correct
    tq.reset_device_errors()
    cache = tq.Cache.allocate(w.B, w.Hkv, w.T, w.k_bits, w.v_bits, w.qjl_m)
    tq.quantize(params, K, V, cache)
    torch.cuda.synchronize()
    assert tq.quantize_device_errors() == 0
    compare_quantized(w, cache, Kh, Vh, 0)
    out = tq.decode_attn(params, W.make_queries(w, device="cuda"), cache, w.T)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and tq.decode_device_errors() == 0
