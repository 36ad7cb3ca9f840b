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


def compare_rows(w: W.Workload, cache: tq.Cache, kx, vx, bi, hi, ti) -> dict:
    """Compare the GPU cache rows (bi, hi, ti) (index arrays) with the oracle's quantization of
    the exact float64 input vectors kx, vx ([n, 128]) under the comparison rules; asserts them and
    returns counts (coordinates, exempt cases, in-band differences)."""
    Pi, S = W.rotation_for(w), W.qjl_for(w)
    kx, vx = np.asarray(kx, np.float64), np.asarray(vx, np.float64)
    kq = O.quantize_vectors(kx, Pi, w.k_bits, S)
    vq = O.quantize_vectors(vx, Pi, w.v_bits, None)
    dev = cache.k_codes.device
    ib, ih, it = (torch.as_tensor(np.asarray(x), device=dev) for x in (bi, hi, ti))
    g = lambda t: t[ib, ih, it].cpu().numpy()
    k_codes, v_codes = g(cache.k_codes), g(cache.v_codes)
    k_norm, v_norm = g(cache.k_norm), g(cache.v_norm)
    k_ex = O.code_exempt(kq["u"], w.k_bits)
    v_ex = O.code_exempt(vq["u"], w.v_bits)
    k_rows_clean = ~k_ex.any(1)
    v_rows_clean = ~v_ex.any(1)
    # rows with no exempt coordinate must be byte-identical to the oracle's packing
    k_want = O.pack_codes(kq["idx"], w.k_bits, O.k_slot_of_coord)
    v_want = O.pack_codes(vq["idx"], w.v_bits, O.v_slot_of_coord)
    kb = np.flatnonzero(~np.all(k_codes == k_want, axis=1) & k_rows_clean)
    vb = np.flatnonzero(~np.all(v_codes == v_want, axis=1) & v_rows_clean)
    assert kb.size == 0, f"key code rows differ from the oracle at {kb[:5]}"
    assert vb.size == 0, f"value code rows differ from the oracle at {vb[:5]}"
    # rows with an exempt coordinate: every other coordinate must match
    k_in_band = v_in_band = 0
    if (~k_rows_clean).any():
        r = ~k_rows_clean
        got = O.unpack_codes(k_codes[r], w.k_bits, O.k_slot_of_coord)
        diff = got != kq["idx"][r]
        assert not (diff & ~k_ex[r]).any(), "key codes differ outside the exemption band"
        k_in_band = int(diff.sum())
    if (~v_rows_clean).any():
        r = ~v_rows_clean
        got = O.unpack_codes(v_codes[r], w.v_bits, O.v_slot_of_coord)
        diff = got != vq["idx"][r]
        assert not (diff & ~v_ex[r]).any(), "value codes differ outside the exemption band"
        v_in_band = int(diff.sum())
    # Stored norms: the bf16 path sums the 128 exact squares in fp32 (chains of 8 fmas, then a
    # 4-level tree: relative error <= 11 * 2^-24 on ||x||^2, 5.5 * 2^-24 on ||x||), takes a
    # correctly rounded sqrt (<= 2^-24) and is compared with the oracle's fp32 rounding of the exact
    # norm (<= 2^-24): |diff| <= 7.5 * 2^-24 * ||x|| <= 7.5 ulp.
    assert ulp_distance_f32(k_norm, kq["n"].astype(np.float32)).max() <= NORM_ULP
    assert ulp_distance_f32(v_norm, vq["n"].astype(np.float32)).max() <= NORM_ULP
    out = {"vectors": int(kx.shape[0]), "coords": int(kq["idx"].size + vq["idx"].size),
           "exempt_codes": int(k_ex.sum() + v_ex.sum()),
           "code_mismatch_in_band": k_in_band + v_in_band}
    if w.qjl_m:
        k_signs = g(cache.k_signs)
        s_ex = O.sign_exempt(kq["sproj"], k_ex)
        s_rows_clean = ~s_ex.any(1)
        s_want = O.pack_signs(kq["signs"])
        sb = np.flatnonzero(~np.all(k_signs == s_want, axis=1) & s_rows_clean)
        assert sb.size == 0, f"sign rows differ from the oracle at {sb[:5]}"
        s_in_band = 0
        if (~s_rows_clean).any():
            r = ~s_rows_clean
            diff = O.unpack_signs(k_signs[r]) != kq["signs"][r]
            assert not (diff & ~s_ex[r]).any(), "sign bits differ outside the exemption band"
            s_in_band = int(diff.sum())
        rn = g(cache.k_rnorm).astype(np.float64)
        ref = kq["rnorm"]
        clean = k_rows_clean
        err = np.abs(rn - ref)[clean]
        assert (err <= 1e-5 * ref[clean] + 1e-30).all(), (err / np.maximum(ref[clean], 1e-30)).max()
        out["sign_bits"] = int(kq["signs"].size)
        out["exempt_signs"] = int(s_ex.sum())
        out["near_zero_signs"] = int((np.abs(kq["sproj"]) <= O.SIGN_BAND).sum())
        out["sign_mismatch_in_band"] = s_in_band
    return out


def merge_counts(total: dict, part: dict) -> dict:
    for k, v in part.items():
        total[k] = total.get(k, 0) + v
    return total


def compare_quantized(w: W.Workload, cache: tq.Cache, Kh, Vh, t_offset: int, rows=None) -> dict:
    """Compare GPU cache rows with the oracle's quantization of the exact inputs.

    Kh, Vh: float64 [B, H, T, 128] inputs written at cache rows [t_offset, t_offset + T); or, with
    rows = [(b, h, t), ...], float64 [len(rows), 128] input vectors for exactly those rows.
    Returns counts; asserts the comparison rules."""
    if rows is None:
        B, H, T, _ = Kh.shape
        bi, hi, ti = (a.reshape(-1) for a in np.meshgrid(np.arange(B), np.arange(H), np.arange(T),
                                                         indexing="ij"))
        kx = np.asarray(Kh, np.float64).reshape(-1, Kh.shape[-1])
        vx = np.asarray(Vh, np.float64).reshape(-1, Vh.shape[-1])
    else:
        bi = np.array([r[0] for r in rows])
        hi = np.array([r[1] for r in rows])
        ti = np.array([r[2] for r in rows])
        kx, vx = np.asarray(Kh, np.float64), np.asarray(Vh, np.float64)
    return compare_rows(w, cache, kx, vx, bi, hi, ti + t_offset)


def compare_full_cache(w: W.Workload, cache: tq.Cache, K: torch.Tensor, V: torch.Tensor,
                       chunk_rows: int = 1 << 16) -> dict:
    """Every row of a cache quantized from the device tensors K, V ([B, Hkv, T, 128], written at
    rows 0..T-1) against the oracle, in chunks of rows; returns the summed counts."""
    B, H, T, d = K.shape
    Kf = K.reshape(B * H * T, d)
    Vf = V.reshape(B * H * T, d)
    total: dict = {}
    for r0 in range(0, B * H * T, chunk_rows):
        r1 = min(B * H * T, r0 + chunk_rows)
        flat = np.arange(r0, r1)
        bi, rem = np.divmod(flat, H * T)
        hi, ti = np.divmod(rem, T)
        kx = Kf[r0:r1].double().cpu().numpy()
        vx = Vf[r0:r1].double().cpu().numpy()
        merge_counts(total, compare_rows(w, cache, kx, vx, bi, hi, ti))
    return total


def exemption_free_inputs(w: W.Workload, spare: int = 64, mixed=None):
    """K, V of the workload's recipe ([B, Hkv, T, 128], input dtype, CPU) in which no vector has a
    coordinate within the code band of a threshold or a sketch value within the sign band of 0:
    the recipe is drawn with T + spare tokens and, per (batch, kv-head), the first T vectors whose
    K and V are both free of exempt cases are kept (about 0.3% of vectors are skipped).  On such
    inputs the cache has exactly one correct value, so a GPU-written cache and the decode over it
    can be compared with the oracle without exceptions.  mixed = (outlier channels, block
    rotation): the exemptions of the mixed layout instead."""
    big = w.scaled(T=w.T + spare)
    K = W.make_kv(big, "k")
    V = W.make_kv(big, "v")
    Pi, S = W.rotation_for(w), W.qjl_for(w)
    Ko = torch.empty((w.B, w.Hkv, w.T, w.head_dim), dtype=K.dtype)
    Vo = torch.empty_like(Ko)
    for b in range(w.B):
        for h in range(w.Hkv):
            if mixed is None:
                kq = O.quantize_vectors(K[b, h].double().numpy(), Pi, w.k_bits, S)
                vq = O.quantize_vectors(V[b, h].double().numpy(), Pi, w.v_bits, None)
                bad = O.code_exempt(kq["u"], w.k_bits).any(1) | O.code_exempt(vq["u"], w.v_bits).any(1)
            else:
                oc, P = mixed
                kq = O.quantize_vectors_mixed(K[b, h].double().numpy(), P, oc, 4, 3, S)
                vq = O.quantize_vectors_mixed(V[b, h].double().numpy(), P, oc, 4, 3, None)
                bad = O.code_exempt_mixed(kq["u"], 4, 3).any(1) | O.code_exempt_mixed(vq["u"], 4, 3).any(1)
            if S is not None:
                bad |= (np.abs(kq["sproj"]) <= O.SIGN_BAND).any(1)
            keep = np.flatnonzero(~bad)[: w.T]
            assert keep.size == w.T, "too few exemption-free vectors in the spare draw"
            Ko[b, h] = K[b, h, torch.as_tensor(keep)]
            Vo[b, h] = V[b, h, torch.as_tensor(keep)]
    return Ko, Vo


def mixed_setup(w: W.Workload):
    """Constants of the outlier-aware mixed layout for a workload: outlier channels from its
    scale draw, the block rotation of those channels, the sketch."""
    oc = W.outlier_channels_for(w)
    return oc, W.make_block_rotation(1000 + w.seed, oc), W.qjl_for(w)


def compare_rows_mixed(w: W.Workload, cache: tq.Cache, kx, vx, bi, hi, ti, oc, P) -> dict:
    """compare_rows for the mixed layout (4-bit outlier half, 3-bit other half): codes, signs,
    both norms of each row and ||r|| against the oracle's mixed quantization."""
    S = W.qjl_for(w)
    kx, vx = np.asarray(kx, np.float64), np.asarray(vx, np.float64)
    kq = O.quantize_vectors_mixed(kx, P, oc, 4, 3, S)
    vq = O.quantize_vectors_mixed(vx, P, oc, 4, 3, None)
    dev = cache.k_codes.device
    ib, ih, it = (torch.as_tensor(np.asarray(x), device=dev) for x in (bi, hi, ti))
    g = lambda t: t[ib, ih, it].cpu().numpy()
    out = {"vectors": int(kx.shape[0]), "coords": int(2 * kx.shape[0] * 128)}
    for name, q, codes, slot in (("k", kq, g(cache.k_codes), O.k_slot_of_coord_mixed),
                                 ("v", vq, g(cache.v_codes), O.v_slot_of_coord_mixed)):
        ex = O.code_exempt_mixed(q["u"], 4, 3)
        got = O.unpack_codes_mixed(codes, 4, 3, slot)
        diff = got != q["idx"]
        assert not (diff & ~ex).any(), f"{name} codes differ outside the exemption band at {np.argwhere(diff & ~ex)[:5]}"
        clean = ~ex.any(1)
        assert np.array_equal(codes[clean], O.pack_codes_mixed(q["idx"], 4, 3, slot)[clean])
        out[name + "_exempt"] = int(ex.sum())
        out[name + "_mismatch_in_band"] = int(diff.sum())
        norms = g(cache.k_norm if name == "k" else cache.v_norm)
        assert ulp_distance_f32(norms[:, 0], q["n_O"].astype(np.float32)).max() <= NORM_ULP
        assert ulp_distance_f32(norms[:, 1], q["n_R"].astype(np.float32)).max() <= NORM_ULP
    k_ex = O.code_exempt_mixed(kq["u"], 4, 3)
    s_ex = O.sign_exempt(kq["sproj"], k_ex)
    signs = O.unpack_signs(g(cache.k_signs))
    sd = signs != kq["signs"]
    assert not (sd & ~s_ex).any(), f"sign bits differ outside the exemption band at {np.argwhere(sd & ~s_ex)[:5]}"
    rn = g(cache.k_rnorm).astype(np.float64)
    clean = ~k_ex.any(1)
    err = np.abs(rn - kq["rnorm"])[clean]
    assert (err <= 1e-5 * kq["rnorm"][clean] + 1e-30).all(), (err / np.maximum(kq["rnorm"][clean], 1e-30)).max()
    out["exempt_codes"] = out["k_exempt"] + out["v_exempt"]
    out["exempt_signs"] = int(s_ex.sum())
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
           "params_for", "compare_rows", "compare_quantized", "compare_full_cache", "merge_counts",
           "mixed_setup", "compare_rows_mixed",
           "exemption_free_inputs", "attention_errors", "assert_attention_close",
           "oracle_cache_arrays", "math", "torch"]
