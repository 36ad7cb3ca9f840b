"""GPU parity of the outlier-aware mixed layout (3.5 bits: the outlier half of the channels at 4
bits, the other half at 3; pages: tproger.ru section on TheTom's llama.cpp fork, turbo3 = 3.5-bit;
ai-manual.ru M5 Max benchmark, per-layer outlier-aware 3/4-bit) through the C ABI, against the
oracle's mixed functions: quantize element by element (bf16 and fp32 inputs, several tiles, ragged
tails, an offset), decode over the oracle's cache (four and eight heads per kv-head, ragged
lengths), and quantize -> decode through the GPU-written cache on inputs free of exempt cases."""
import numpy as np
import pytest
import torch

import decode_attention_11_b200 as tq
import workloads as W
from oracle import tq_oracle as O

from _parity import (assert_attention_close, compare_rows_mixed, exemption_free_inputs, gpu_inputs,
                     mixed_setup)

pytestmark = pytest.mark.gpu

CASES = {
    "llama3_8b_128k_b4": dict(T=531, B=2, Hkv=2, Hq=8),     # 4 heads per kv-head
    "moe_1m": dict(T=700, B=1, Hkv=2, Hq=16),                # 8 heads per kv-head
    "single_head_4k": dict(T=400, B=1, Hkv=1, Hq=4),         # fp32 inputs
}


def _mixed(name, **over):
    w = W.CONFIGS[name].scaled(**{**CASES[name], **over})
    oc, P, S = mixed_setup(w)
    params = tq.Params.create(P, S, 4, 4, outlier_channels=oc)
    return w, oc, P, S, params


def _rows(B, H, T, t_off=0):
    bi, hi, ti = (a.reshape(-1) for a in np.meshgrid(np.arange(B), np.arange(H), np.arange(T), indexing="ij"))
    return bi, hi, ti + t_off


@pytest.mark.parametrize("name", list(CASES))
def test_mixed_quantize_parity(name):
    w, oc, P, S, params = _mixed(name)
    K, V, Kh, Vh = gpu_inputs(w)
    t_off = 11
    cache = tq.Cache.allocate(w.B, w.Hkv, w.T + t_off + 3, 4, 4, w.qjl_m, layout=tq.TQ_LAYOUT_MIXED)
    tq.quantize(params, K, V, cache, t_offset=t_off)
    torch.cuda.synchronize()
    assert tq.quantize_device_errors() == 0
    st = compare_rows_mixed(w, cache, Kh.reshape(-1, 128), Vh.reshape(-1, 128),
                            *_rows(w.B, w.Hkv, w.T, t_off), oc, P)
    print(f"{name} mixed: {st['exempt_codes']} exempt codes of {st['coords']}, "
          f"{st['k_mismatch_in_band'] + st['v_mismatch_in_band']} differ")
    for arr in (cache.k_codes, cache.v_codes, cache.k_norm, cache.v_norm):
        a = arr.cpu()
        assert a[:, :, :t_off].abs().sum() == 0 and a[:, :, t_off + w.T:].abs().sum() == 0


@pytest.mark.parametrize("name", ["llama3_8b_128k_b4", "moe_1m"])
def test_mixed_decode_parity(name):
    w, oc, P, S, params = _mixed(name)
    K, V, Kh, Vh = gpu_inputs(w)
    c = O.quantize_cache_mixed(Kh, Vh, P, oc, (4, 3), (4, 3), S)
    arrays = {k: c[k] for k in ("k_codes", "k_signs", "k_norm", "k_rnorm", "v_codes", "v_norm")}
    cache = tq.Cache.from_arrays(arrays, 4, 4, w.qjl_m, layout=tq.TQ_LAYOUT_MIXED)
    q = W.make_queries(w)
    for L in (w.T, w.T - 37, 65, 16, 1):
        out = tq.decode_attn(params, q.cuda(), cache, L)
        torch.cuda.synchronize()
        ref = O.decode_attention_mixed(q.double().numpy(), P, S, c, (4, 3), (4, 3), L)
        assert_attention_close(out.cpu().numpy(), ref)
    assert tq.decode_device_errors() == 0


def test_mixed_quantize_then_decode_end_to_end():
    """GPU quantize, then GPU decode over the GPU-written mixed cache, against the oracle's; the
    inputs have no exempt case in either half, so the cache has one correct value."""
    w, oc, P, S, params = _mixed("llama3_8b_128k_b4")
    K, V = exemption_free_inputs(w, mixed=(oc, P))
    Kh, Vh = K.double().numpy(), V.double().numpy()
    kq = O.quantize_vectors_mixed(Kh.reshape(-1, 128), P, oc, 4, 3, S)
    vq = O.quantize_vectors_mixed(Vh.reshape(-1, 128), P, oc, 4, 3, None)
    bad = (O.code_exempt_mixed(kq["u"], 4, 3).any(1) | O.code_exempt_mixed(vq["u"], 4, 3).any(1)
           | (np.abs(kq["sproj"]) <= O.SIGN_BAND).any(1))
    assert not bad.any(), "mixed-layout exemption in the test data: choose another draw"
    cache = tq.Cache.allocate(w.B, w.Hkv, w.T, 4, 4, w.qjl_m, layout=tq.TQ_LAYOUT_MIXED)
    tq.quantize(params, K.cuda(), V.cuda(), cache)
    q = W.make_queries(w)
    out = tq.decode_attn(params, q.cuda(), cache, w.T).cpu().numpy()
    torch.cuda.synchronize()
    compare_rows_mixed(w, cache, Kh.reshape(-1, 128), Vh.reshape(-1, 128), *_rows(w.B, w.Hkv, w.T), oc, P)
    c = O.quantize_cache_mixed(Kh, Vh, P, oc, (4, 3), (4, 3), S)
    ref = O.decode_attention_mixed(q.double().numpy(), P, S, c, (4, 3), (4, 3), w.T)
    assert_attention_close(out, ref)


def test_mixed_full_size_quantize_and_decode():
    """The 128K batch-4 layer at full size in the mixed layout: every quantized row of one
    (batch, kv-head) slice against the oracle, and decode over a slice the oracle wrote."""
    w = W.CONFIGS["llama3_8b_128k_b4"]
    oc, P, S = mixed_setup(w)
    params = tq.Params.create(P, S, 4, 4, outlier_channels=oc)
    K = W.make_kv(w, "k", device="cuda")
    V = W.make_kv(w, "v", device="cuda")
    cache = tq.Cache.allocate(w.B, w.Hkv, w.T, 4, 4, w.qjl_m, layout=tq.TQ_LAYOUT_MIXED)
    tq.quantize(params, K, V, cache)
    torch.cuda.synchronize()
    assert tq.quantize_device_errors() == 0
    b, kvh = w.B - 1, w.Hkv - 1
    Kh = K[b:b + 1, kvh:kvh + 1].double().cpu().numpy()
    Vh = V[b:b + 1, kvh:kvh + 1].double().cpu().numpy()
    del K, V
    tot = {"exempt_codes": 0, "coords": 0}
    for t0 in range(0, w.T, 1 << 15):
        t1 = min(w.T, t0 + (1 << 15))
        n = t1 - t0
        st = compare_rows_mixed(w, cache, Kh[0, 0, t0:t1], Vh[0, 0, t0:t1], np.full(n, b), np.full(n, kvh),
                                np.arange(t0, t1), oc, P)
        tot["exempt_codes"] += st["exempt_codes"]
        tot["coords"] += st["coords"]
    print(f"mixed full size, one slice: exempt fraction {tot['exempt_codes'] / tot['coords']:.3e}")
    assert tot["exempt_codes"] / tot["coords"] <= 1e-5
    c = O.quantize_cache_mixed(Kh, Vh, P, oc, (4, 3), (4, 3), S)
    for key in ("k_codes", "k_signs", "k_norm", "k_rnorm", "v_codes", "v_norm"):
        getattr(cache, key)[b, kvh].copy_(torch.as_tensor(c[key][0, 0]))
    q = W.make_queries(w, device="cuda")
    out = tq.decode_attn(params, q, cache, w.T)
    torch.cuda.synchronize()
    heads = list(range(kvh * w.group, (kvh + 1) * w.group))
    ref = O.decode_attention_mixed(q[b:b + 1, heads].double().cpu().numpy(), P, S,
                                   {k: v for k, v in c.items()}, (4, 3), (4, 3), w.T)[0]
    assert_attention_close(out[b, heads].cpu().numpy(), ref)
