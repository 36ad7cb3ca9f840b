"""Comparison helpers for GPU-vs-oracle parity tests (test infrastructure)."""
import math

import numpy as np
import torch

import decode_attention_11_b200 as tq
import workloads as W
from oracle import tq_oracle as O

ATTN_MAX_ABS = 2e-3   # decode attention: max-abs error vs the float64 oracle
ATTN_REL_L2 = 1e-3    # decode attention: relative L2 error vs the float64 oracle
EXEMPT_FRACTION_MAX = 1e-5
NORM_ULP = 8          # stored ||x|| vs the oracle's float32 rounding of the exact norm


def ulp_distance_f32(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    ia = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    ib = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(ia - ib)


def gpu_inputs(w: W.Workload, device="cuda"):
    """K, V on the device plus their exact float64 host copies."""
    K = W.make_kv(w, "k", device="cpu")
    V = W.make_kv(w, "v", device="cpu")
    return K.to(device), V.to(device), K.double().numpy(), V.double().numpy()


def params_for(w: W.Workload, device="cuda") -> tq.Params:
    return tq.Params.create(W.rotation_for(w), W.qjl_for(w), w.k_bits, w.v_bits, device=device)


def compare_quantized(w: W.Workload, cache: tq.Cache, Kh, Vh, t_offset: int, rows=None) -> dict:
    """Compare GPU cache rows with the oracle's quantization of the exact inputs.

    Kh, Vh: float64 [B, H, T, 128] inputs written at cache rows [t_offset, t_offset + T); or, with
    rows = [(b, h, t), ...], float64 [len(rows), 128] input vectors for exactly those rows.
    Returns counts; asserts the comparison rules."""
    Pi, S = W.rotation_for(w), W.qjl_for(w)
    if rows is None:
        B, H, T, _ = Kh.shape
        rows = [(b, h, t) for b in range(B) for h in range(H) for t in range(T)]
        bi = np.array([r[0] for r in rows])
        hi = np.array([r[1] for r in rows])
        ti = np.array([r[2] for r in rows])
        kx = Kh[bi, hi, ti]
        vx = Vh[bi, hi, ti]
    else:
        bi = np.array([r[0] for r in rows])
        hi = np.array([r[1] for r in rows])
        ti = np.array([r[2] for r in rows])
        kx, vx = np.asarray(Kh, np.float64), np.asarray(Vh, np.float64)
    kq = O.quantize_vectors(kx, Pi, w.k_bits, S)
    vq = O.quantize_vectors(vx, Pi, w.v_bits, None)
    tc = ti + t_offset
    dev = cache.k_codes.device
    ib, ih, it = (torch.as_tensor(x, device=dev) for x in (bi, hi, tc))
    g = lambda t: t[ib, ih, it].cpu().numpy()
    k_codes, v_codes = g(cache.k_codes), g(cache.v_codes)
    k_norm, v_norm = g(cache.k_norm), g(cache.v_norm)
    k_idx = O.unpack_codes(k_codes, w.k_bits, O.k_slot_of_coord)
    v_idx = O.unpack_codes(v_codes, w.v_bits, O.v_slot_of_coord)
    k_ex = O.code_exempt(kq["u"], w.k_bits)
    v_ex = O.code_exempt(vq["u"], w.v_bits)
    k_bad = (k_idx != kq["idx"]) & ~k_ex
    v_bad = (v_idx != vq["idx"]) & ~v_ex
    assert not k_bad.any(), f"key codes differ outside the exemption band at {np.argwhere(k_bad)[:5]}"
    assert not v_bad.any(), f"value codes differ outside the exemption band at {np.argwhere(v_bad)[:5]}"
    # rows with no exempt coordinate must be byte-identical to the oracle's packing
    k_rows_clean = ~k_ex.any(1)
    v_rows_clean = ~v_ex.any(1)
    assert np.array_equal(k_codes[k_rows_clean], O.pack_codes(kq["idx"], w.k_bits, O.k_slot_of_coord)[k_rows_clean])
    assert np.array_equal(v_codes[v_rows_clean], O.pack_codes(vq["idx"], w.v_bits, O.v_slot_of_coord)[v_rows_clean])
    # Stored norms: the bf16 path sums the 128 exact squares in fp32 (chains of 8 fmas, then a
    # 4-level tree: relative error <= 11 * 2^-24 on ||x||^2, 5.5 * 2^-24 on ||x||), takes a
    # correctly rounded sqrt (<= 2^-24) and is compared with the oracle's fp32 rounding of the exact
    # norm (<= 2^-24): |diff| <= 7.5 * 2^-24 * ||x|| <= 7.5 ulp.
    assert ulp_distance_f32(k_norm, kq["n"].astype(np.float32)).max() <= NORM_ULP
    assert ulp_distance_f32(v_norm, vq["n"].astype(np.float32)).max() <= NORM_ULP
    out = {"coords": k_idx.size + v_idx.size,
           "exempt_codes": int(k_ex.sum() + v_ex.sum()),
           "code_mismatch_in_band": int(((k_idx != kq["idx"]) & k_ex).sum() + ((v_idx != vq["idx"]) & v_ex).sum())}
    if w.qjl_m:
        signs = O.unpack_signs(g(cache.k_signs))
        s_ex = O.sign_exempt(kq["sproj"], k_ex)
        s_bad = (signs != kq["signs"]) & ~s_ex
        assert not s_bad.any(), f"sign bits differ outside the exemption band at {np.argwhere(s_bad)[:5]}"
        rn = g(cache.k_rnorm).astype(np.float64)
        ref = kq["rnorm"]
        clean = ~k_ex.any(1)
        err = np.abs(rn - ref)[clean]
        assert (err <= 1e-5 * ref[clean] + 1e-30).all(), (err / np.maximum(ref[clean], 1e-30)).max()
        out["exempt_signs"] = int(s_ex.sum())
        out["sign_mismatch_in_band"] = int(((signs != kq["signs"]) & s_ex).sum())
    return out


def attention_errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    max_abs = float(np.max(np.abs(got - ref))) if got.size else 0.0
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)) if got.size else 0.0
    return max_abs, rel


def assert_attention_close(got, ref):
    max_abs, rel = attention_errors(got, ref)
    assert max_abs <= ATTN_MAX_ABS and (rel <= ATTN_REL_L2 or np.linalg.norm(ref) == 0), (max_abs, rel)
    return max_abs, rel


def oracle_cache_arrays(w: W.Workload, Kh, Vh, T_cap=None):
    """Packed cache built by the oracle from exact inputs, padded to T_cap rows."""
    Pi, S = W.rotation_for(w), W.qjl_for(w)
    c = O.quantize_cache(Kh, Vh, Pi, w.k_bits, w.v_bits, S)
    B, H, T, _ = Kh.shape
    T_cap = T if T_cap is None else T_cap
    pad = lambda a: np.concatenate([a, np.zeros((B, H, T_cap - T) + a.shape[3:], a.dtype)], axis=2)
    keys = ["k_codes", "k_norm", "v_codes", "v_norm"] + (["k_signs", "k_rnorm"] if S is not None else [])
    return {k: pad(c[k]) for k in keys}, c


__all__ = ["ATTN_MAX_ABS", "ATTN_REL_L2", "EXEMPT_FRACTION_MAX", "ulp_distance_f32", "gpu_inputs",
           "params_for", "compare_quantized", "attention_errors", "assert_attention_close",
           "oracle_cache_arrays", "math", "torch"]
