"""CPU oracle for TurboQuant-style KV-cache compression and decode attention.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain, float64 statement
of what the CUDA path computes.  Only the test-suite, ``__graft_entry__.smoke``
and the CPU-baseline leg of ``bench.py`` may import it.  It shares no code with
the library (``decode_attention_11_b200``) and never imports it; the only
module both sides use is ``workloads`` (seeded random inputs).

Sources (all page citations name the page and the passage):

* ai-news.ru overview of TurboQuant ("When Google published the paper on the
  memory-compression algorithm..."), paragraph on the "first idea" and the
  "second": each vector is multiplied by a random orthogonal matrix so its
  coordinates become near-independent and near-Gaussian, and a Lloyd-Max grid
  precomputed once for that known distribution quantizes every coordinate;
  the codebook is static and needs no calibration.  Same page, next
  paragraph: the "third component", a 1-bit QJL correction of the residual.
* tproger.ru, "Google TurboQuant in simple words", section "Step 1:
  PolarQuant": the rotation precedes quantization, and Lloyd-Max is applied
  to each coordinate independently with no extra bits for quantization
  parameters.  Section "Step 2: QJL": a Johnson-Lindenstrauss sketch spends
  one extra bit to make the residual error unbiased.  Section "Benchmarks --
  from independent implementations": TQ3 MSE 0.034, TQ4 MSE 0.009, a TQ3
  block is 52 bytes per 128 values.
* The QJL estimator of the inner product (the unbiased 1-bit residual
  correction of tproger.ru "Step 2: QJL" and the ai-news.ru third component):
  <q,k> ~= <q,k_mse> + ||r|| sqrt(pi/2)/m <S q, sign(S r)> with a Gaussian S
  of m rows, storing sign(S r) and ||r||.

Readings taken where the pages are silent:

* the Lloyd-Max density is the standard normal (rotated, rescaled
  coordinates u = sqrt(d) * Pi x / ||x||);
* stored centroids are the Lloyd-Max centroids rounded to the nearest fp16,
  thresholds are the exact midpoints of adjacent stored centroids;
* an index counts the thresholds at or below the value (a tie goes up);
* one fp32 norm ||x|| per vector; the QJL residual is taken in the rotated,
  normalized basis (rho = u - c[idx]), ||r|| = ||x|| ||rho|| / sqrt(d), and a
  sign bit is 1 when (S rho)_l >= 0;
* QJL applies to keys only; values carry codes and a norm;
* decode uses scale 1/sqrt(d), attends to all seq_len tokens, GQA head h reads
  kv-head h // (Hq/Hkv), and an empty context gives a zero output;
* the packed row layouts below (bit streams in a fixed slot order).

Parity status: every function here is pinned by tests in
``tests/test_oracle_pins.py`` (closed forms, Lloyd conditions, bounds, the
pages' printed figures, brute force on tiny inputs, QJL unbiasedness).
"""
from __future__ import annotations

import math
from statistics import NormalDist
from typing import Dict, Optional

import numpy as np

D = 128  # head_dim fixed by the method's configurations
SQRT_PI_OVER_2 = math.sqrt(math.pi / 2.0)


# ---------------------------------------------------------------------------
# Lloyd-Max codebook for N(0,1)   (ai-news.ru overview, the "second idea")
# ---------------------------------------------------------------------------

def _pdf(x: float) -> float:
    if math.isinf(x):
        return 0.0
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _cdf(x: float) -> float:
    if x == math.inf:
        return 1.0
    if x == -math.inf:
        return 0.0
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def lloyd_max_gaussian(bits: int, max_iter: int = 100000, tol: float = 1e-13):
    """Lloyd iteration on the standard normal density.

    Start at the quantiles (k + 1/2) / 2^b; alternate the two Lloyd
    conditions -- each threshold is the midpoint of its neighbouring
    centroids, each centroid is the conditional mean E[X | t_{k-1} <= X < t_k]
    = (phi(t_{k-1}) - phi(t_k)) / (Phi(t_k) - Phi(t_{k-1})) -- until the
    largest centroid move is below ``tol``; then make the solution exactly
    symmetric (c_{L-1-k} = -c_k).

    Returns (centroids float64[L], thresholds float64[L-1], distortion, iterations),
    distortion = E[(X - Q(X))^2] = 1 - sum_k P_k c_k^2 (centroid condition).
    """
    if not 1 <= bits <= 8:
        raise ValueError("bits must be in 1..8")
    L = 1 << bits
    nd = NormalDist()
    c = [nd.inv_cdf((k + 0.5) / L) for k in range(L)]
    it = 0
    for it in range(1, max_iter + 1):
        t = [-math.inf] + [0.5 * (c[i] + c[i + 1]) for i in range(L - 1)] + [math.inf]
        new = [(_pdf(t[k]) - _pdf(t[k + 1])) / (_cdf(t[k + 1]) - _cdf(t[k])) for k in range(L)]
        move = max(abs(a - b) for a, b in zip(c, new))
        c = new
        if move < tol:
            break
    c = np.array(c, dtype=np.float64)
    c = 0.5 * (c - c[::-1])  # exact symmetry
    t = 0.5 * (c[:-1] + c[1:])
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    P = np.array([_cdf(edges[k + 1]) - _cdf(edges[k]) for k in range(L)])
    distortion = 1.0 - float(np.sum(P * c * c))
    return c, t, distortion, it


class Codebook:
    """Stored codebook: fp16-representable centroids, fp32 midpoint thresholds."""

    def __init__(self, bits: int):
        c, _, dist, _ = lloyd_max_gaussian(bits)
        self.bits = bits
        self.lloyd_centroids = c
        self.lloyd_distortion = dist
        c16 = c.astype(np.float16).astype(np.float64)
        self.centroids = c16  # float64 holding fp16 values
        t = 0.5 * (c16[:-1] + c16[1:])
        assert np.all(t.astype(np.float32).astype(np.float64) == t), "midpoints exact in fp32"
        self.thresholds = t

    @property
    def levels(self) -> int:
        return 1 << self.bits


_CODEBOOKS: Dict[int, Codebook] = {}


def codebook(bits: int) -> Codebook:
    if bits not in _CODEBOOKS:
        _CODEBOOKS[bits] = Codebook(bits)
    return _CODEBOOKS[bits]


def quantize_index(u: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """idx = #{i : u >= t_i} (a value equal to a threshold goes to the upper cell)."""
    return (u[..., None] >= thresholds).sum(axis=-1).astype(np.int64)


# ---------------------------------------------------------------------------
# Quantize (tproger.ru "Step 1: PolarQuant" + "Step 2: QJL")
# ---------------------------------------------------------------------------

def quantize_vectors(X: np.ndarray, Pi: np.ndarray, k_bits: int,
                     S: Optional[np.ndarray] = None) -> dict:
    """Compress N vectors x (rows of X, any float dtype, taken exactly in float64).

    n = ||x||;  u = sqrt(d) * Pi x / n  (u = 0 when n = 0);
    idx_j = #{i : u_j >= t_i};  rho = u - c[idx];
    with S (QJL):  ||r|| = n ||rho|| / sqrt(d),  sign_l = [(S rho)_l >= 0].
    """
    X = np.asarray(X, dtype=np.float64)
    Pi = np.asarray(Pi, dtype=np.float64)
    d = X.shape[-1]
    cb = codebook(k_bits)
    n = np.sqrt(np.sum(X * X, axis=-1))
    Y = X @ Pi.T
    safe = np.where(n > 0, n, 1.0)
    u = np.where((n > 0)[:, None], math.sqrt(d) * Y / safe[:, None], 0.0)
    idx = quantize_index(u, cb.thresholds)
    rho = u - cb.centroids[idx]
    out = {"n": n, "u": u, "idx": idx, "rho": rho}
    if S is not None:
        S = np.asarray(S, dtype=np.float64)
        out["rnorm"] = n * np.sqrt(np.sum(rho * rho, axis=-1)) / math.sqrt(d)
        sproj = rho @ S.T
        out["sproj"] = sproj
        out["signs"] = (sproj >= 0).astype(np.int64)
    return out


# ---------------------------------------------------------------------------
# Packed row layouts (the pages give none; the layout below is a reading)
# ---------------------------------------------------------------------------

def k_slot_of_coord(j: int) -> int:
    """Key-code row: coordinate j = 16*kap + 8*h + 2*tau + eps sits at slot 32*tau + 4*kap + 2*h + eps."""
    kap, rem = divmod(j, 16)
    h, rem = divmod(rem, 8)
    tau, eps = divmod(rem, 2)
    return 32 * tau + 4 * kap + 2 * h + eps


def v_slot_of_coord(j: int) -> int:
    """Value-code row: coordinate j = 8*nu + gam sits at slot 16*gam + nu."""
    nu, gam = divmod(j, 8)
    return 16 * gam + nu


def sign_bit_of_row(l: int) -> int:
    """Sign row: sketch row l = 16*kap + 8*h + 2*tau + eps sits at bit 32*tau + (2*kap + h) + 16*eps."""
    kap, rem = divmod(l, 16)
    h, rem = divmod(rem, 8)
    tau, eps = divmod(rem, 2)
    return 32 * tau + (2 * kap + h) + 16 * eps


def pack_codes(idx: np.ndarray, bits: int, slot_of_coord) -> np.ndarray:
    """Rows of 128 b-bit codes -> bytes[N, 16*b]: slot s holds bits [b*s, b*s+b) of the row,
    least significant first; row bit k is bit (k % 8) of byte k // 8."""
    N, d = idx.shape
    out = np.zeros((N, d * bits // 8), dtype=np.uint8)
    for j in range(d):
        s = slot_of_coord(j)
        for i in range(bits):
            k = bits * s + i
            bit = ((idx[:, j] >> i) & 1).astype(np.uint8)
            out[:, k // 8] |= bit << (k % 8)
    return out


def unpack_codes(rows: np.ndarray, bits: int, slot_of_coord) -> np.ndarray:
    rows = np.asarray(rows, dtype=np.uint8)
    N = rows.shape[0]
    d = rows.shape[1] * 8 // bits
    idx = np.zeros((N, d), dtype=np.int64)
    for j in range(d):
        s = slot_of_coord(j)
        for i in range(bits):
            k = bits * s + i
            idx[:, j] |= ((rows[:, k // 8] >> (k % 8)) & 1).astype(np.int64) << i
    return idx


def pack_signs(signs: np.ndarray) -> np.ndarray:
    N, m = signs.shape
    out = np.zeros((N, m // 8), dtype=np.uint8)
    for l in range(m):
        k = sign_bit_of_row(l)
        out[:, k // 8] |= (signs[:, l].astype(np.uint8) & 1) << (k % 8)
    return out


def unpack_signs(rows: np.ndarray) -> np.ndarray:
    rows = np.asarray(rows, dtype=np.uint8)
    N = rows.shape[0]
    m = rows.shape[1] * 8
    s = np.zeros((N, m), dtype=np.int64)
    for l in range(m):
        k = sign_bit_of_row(l)
        s[:, l] = (rows[:, k // 8] >> (k % 8)) & 1
    return s


# ---------------------------------------------------------------------------
# Cache construction (quantize K and V of a [B, Hkv, T, d] block)
# ---------------------------------------------------------------------------

def quantize_cache(K: np.ndarray, V: np.ndarray, Pi: np.ndarray, k_bits: int, v_bits: int,
                   S: Optional[np.ndarray]) -> dict:
    """K, V: [B, Hkv, T, d].  Returns the packed cache arrays plus the float64
    intermediates (u, sproj) that the comparison rules need."""
    B, H, T, d = K.shape
    kq = quantize_vectors(K.reshape(-1, d), Pi, k_bits, S)
    vq = quantize_vectors(V.reshape(-1, d), Pi, v_bits, None)
    cache = {
        "k_codes": pack_codes(kq["idx"], k_bits, k_slot_of_coord).reshape(B, H, T, -1),
        "k_norm": kq["n"].astype(np.float32).reshape(B, H, T),
        "v_codes": pack_codes(vq["idx"], v_bits, v_slot_of_coord).reshape(B, H, T, -1),
        "v_norm": vq["n"].astype(np.float32).reshape(B, H, T),
        "k_u": kq["u"].reshape(B, H, T, d),
        "k_idx": kq["idx"].reshape(B, H, T, d),
        "v_u": vq["u"].reshape(B, H, T, d),
        "v_idx": vq["idx"].reshape(B, H, T, d),
    }
    if S is not None:
        cache["k_signs"] = pack_signs(kq["signs"]).reshape(B, H, T, -1)
        cache["k_rnorm"] = kq["rnorm"].astype(np.float32).reshape(B, H, T)
        cache["k_sproj"] = kq["sproj"].reshape(B, H, T, -1)
    return cache


# ---------------------------------------------------------------------------
# Decode attention over the packed cache (float64)
# ---------------------------------------------------------------------------

def score_estimates(q: np.ndarray, Pi: np.ndarray, S: Optional[np.ndarray], k_codes: np.ndarray,
                    k_norm: np.ndarray, k_bits: int, k_signs: Optional[np.ndarray] = None,
                    k_rnorm: Optional[np.ndarray] = None) -> np.ndarray:
    """est_i = <q', khat'_i> + ||r_i|| sqrt(pi/2)/m <S q', 2 sign_i - 1>  for one query and
    T packed key rows.  q' = Pi q;  khat'_i = (n_i / sqrt(d)) c[idx_i]."""
    q = np.asarray(q, dtype=np.float64)
    Pi64 = np.asarray(Pi, dtype=np.float64)
    d = q.shape[-1]
    qp = Pi64 @ q
    idx = unpack_codes(k_codes, k_bits, k_slot_of_coord)
    khat = (np.asarray(k_norm, np.float64)[:, None] / math.sqrt(d)) * codebook(k_bits).centroids[idx]
    est = khat @ qp
    if S is not None:
        S64 = np.asarray(S, dtype=np.float64)
        m = S64.shape[0]
        sq = S64 @ qp
        pm = 2.0 * unpack_signs(k_signs) - 1.0
        est = est + np.asarray(k_rnorm, np.float64) * (SQRT_PI_OVER_2 / m) * (pm @ sq)
    return est


def softmax_weighted_sum(scores: np.ndarray, values: np.ndarray) -> np.ndarray:
    """sum_i softmax(scores)_i values_i; an empty set of tokens gives 0."""
    if scores.shape[0] == 0:
        return np.zeros(values.shape[-1], dtype=np.float64)
    m = np.max(scores)
    w = np.exp(scores - m)
    return (w @ values) / np.sum(w)


def decode_attention(q: np.ndarray, Pi: np.ndarray, S: Optional[np.ndarray], cache: dict,
                     k_bits: int, v_bits: int, seq_len: int, scale: Optional[float] = None,
                     heads=None) -> np.ndarray:
    """Single-token attention of q [B, Hq, d] over the first seq_len tokens of the
    packed cache ([B, Hkv, T, ...] arrays).  Returns float64 [B, Hq, d].

    o'_h = sum_i softmax(scale * est_i)_i (nV_i / sqrt(d)) c_V[idxV_i];  o_h = Pi^T o'_h.
    ``heads`` optionally restricts the (b, h) pairs computed (others stay 0).
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = cache["k_codes"].shape[1]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Pi64 = np.asarray(Pi, dtype=np.float64)
    cV = codebook(v_bits).centroids
    out = np.zeros((B, Hq, d), dtype=np.float64)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    vhat_cache = {}
    for b, h in pairs:
        kv = h // g
        T = seq_len
        sl = (b, kv, slice(0, T))
        est = score_estimates(
            q[b, h], Pi, S, cache["k_codes"][sl], cache["k_norm"][sl], k_bits,
            cache["k_signs"][sl] if S is not None else None,
            cache["k_rnorm"][sl] if S is not None else None)
        if (b, kv) not in vhat_cache:
            vidx = unpack_codes(cache["v_codes"][sl], v_bits, v_slot_of_coord)
            vhat_cache[(b, kv)] = (np.asarray(cache["v_norm"][sl], np.float64)[:, None]
                                   / math.sqrt(d)) * cV[vidx]
        o_rot = softmax_weighted_sum(scale * est, vhat_cache[(b, kv)])
        out[b, h] = Pi64.T @ o_rot
    return out


def exact_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: Optional[float] = None
                    ) -> np.ndarray:
    """Uncompressed softmax(q K^T * scale) V with GQA, float64; q [B,Hq,d], K,V [B,Hkv,T,d]."""
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    B, Hq, d = q.shape
    Hkv = K.shape[1]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((B, Hq, d))
    for b in range(B):
        for h in range(Hq):
            out[b, h] = softmax_weighted_sum(scale * (K[b, h // g] @ q[b, h]), V[b, h // g])
    return out


# ---------------------------------------------------------------------------
# Comparison rules for code/sign bytes (exemptions near decision boundaries)
# ---------------------------------------------------------------------------

CODE_BAND = 1e-6   # |u_j - t_i| <= 1e-6: the rounding of u decides the code
SIGN_BAND = 1e-5   # |(S rho)_l| <= 1e-5 (normalized units): the rounding decides the sign


def code_exempt(u: np.ndarray, bits: int, band: float = CODE_BAND) -> np.ndarray:
    t = codebook(bits).thresholds
    return np.any(np.abs(u[..., None] - t) <= band, axis=-1)


def sign_exempt(sproj: np.ndarray, code_exempt_mask: np.ndarray, band: float = SIGN_BAND
                ) -> np.ndarray:
    vec = np.any(code_exempt_mask, axis=-1, keepdims=True)
    return (np.abs(sproj) <= band) | vec


__all__ = [
    "D", "lloyd_max_gaussian", "Codebook", "codebook", "quantize_index", "quantize_vectors",
    "k_slot_of_coord", "v_slot_of_coord", "sign_bit_of_row", "pack_codes", "unpack_codes",
    "pack_signs", "unpack_signs", "quantize_cache", "score_estimates", "softmax_weighted_sum",
    "decode_attention", "exact_attention", "code_exempt", "sign_exempt", "CODE_BAND", "SIGN_BAND",
]
