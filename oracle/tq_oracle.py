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
# Outlier-aware mixed precision (tproger.ru, section on TheTom's llama.cpp fork: "turbo3" is
# 3.5-bit KV quantization, 4.6x smaller than FP16; ai-manual.ru M5 Max KV-cache benchmark,
# "when TurboQuant is needed": per-layer outlier-aware 3/4-bit quantization)
#
# Reading (the pages give no construction): the head's channels split into two fixed halves,
# an "outlier" half O (a per-layer parameter, 64 channels) coded with bits_O and the other half
# R with bits_R (4 and 3 bits average 3.5).  Each half is an instance of the method's first two
# steps on its own: its own random rotation (the block rotation Pi_blk puts Pi_O x_O in rows
# 0..63 and Pi_R x_R in rows 64..127), its own norm n_g = ||x_g||, coordinates
# u_g = sqrt(64) (Pi_blk x)_g / n_g and its own Lloyd-Max codebook.  The QJL step is unchanged
# but acts on the whole residual in the block-rotated basis,
#     r = Pi_blk x - khat,   khat_g = (n_g / sqrt(64)) c_g[idx_g],
# so the estimator <q,k> ~= <q',khat> + ||r|| sqrt(pi/2)/m <S q', sign(S r)> (q' = Pi_blk q) keeps
# its form.  The sketch value compared with 0 is taken in the units of the plain method,
# sigma = sqrt(128)/||x|| S r (which equals S rho when both halves share one norm).
# ---------------------------------------------------------------------------

HALF = D // 2


def quantize_vectors_mixed(X: np.ndarray, Pi_blk: np.ndarray, outlier_channels, bits_O: int,
                           bits_R: int, S: Optional[np.ndarray] = None) -> dict:
    """Compress N vectors (rows of X, taken exactly in float64) in the mixed layout.

    n_g = ||x restricted to the channels of half g||;  y = Pi_blk x;
    u_g = sqrt(64) y_g / n_g (0 when n_g = 0);  idx_g = #{i : u_g >= t_i of codebook(bits_g)};
    with S: r = y - khat, ||r||, sigma = sqrt(128)/||x|| S r, sign_l = [sigma_l >= 0]."""
    X = np.asarray(X, dtype=np.float64)
    P = np.asarray(Pi_blk, dtype=np.float64)
    O = np.sort(np.asarray(outlier_channels, dtype=np.int64))
    R = np.setdiff1d(np.arange(D), O)
    n = {0: np.sqrt(np.sum(X[:, O] ** 2, axis=-1)), 1: np.sqrt(np.sum(X[:, R] ** 2, axis=-1))}
    Y = X @ P.T
    u = np.zeros_like(Y)
    idx = np.zeros(Y.shape, dtype=np.int64)
    khat = np.zeros_like(Y)
    for g, bits in ((0, bits_O), (1, bits_R)):
        cols = slice(HALF * g, HALF * (g + 1))
        ng = n[g]
        safe = np.where(ng > 0, ng, 1.0)
        u[:, cols] = np.where((ng > 0)[:, None], math.sqrt(HALF) * Y[:, cols] / safe[:, None], 0.0)
        cb = codebook(bits)
        idx[:, cols] = quantize_index(u[:, cols], cb.thresholds)
        khat[:, cols] = (ng[:, None] / math.sqrt(HALF)) * cb.centroids[idx[:, cols]]
    out = {"n_O": n[0], "n_R": n[1], "u": u, "idx": idx, "y": Y, "khat": khat}
    if S is not None:
        S = np.asarray(S, dtype=np.float64)
        r = Y - khat
        out["rnorm"] = np.sqrt(np.sum(r * r, axis=-1))
        nx = np.sqrt(n[0] ** 2 + n[1] ** 2)
        sproj = np.where((nx > 0)[:, None], math.sqrt(D) * (r @ S.T) / np.where(nx > 0, nx, 1.0)[:, None], 0.0)
        out["sproj"] = sproj
        out["signs"] = (sproj >= 0).astype(np.int64)
    return out


def k_slot_of_coord_mixed(j: int) -> int:
    """Mixed key row: half g = j // 64 is its own bit stream (half O first); within it,
    j - 64 g = 16 a + 8 h + 2 tau + eps sits at slot 16 tau + 4 a + 2 h + eps."""
    jj = j % HALF
    a, rem = divmod(jj, 16)
    h, rem = divmod(rem, 8)
    tau, eps = divmod(rem, 2)
    return 16 * tau + 4 * a + 2 * h + eps


def v_slot_of_coord_mixed(j: int) -> int:
    """Mixed value row: within half g, coordinate j - 64 g = 8 nu + gam sits at slot 8 gam + nu."""
    nu, gam = divmod(j % HALF, 8)
    return 8 * gam + nu


def pack_codes_mixed(idx: np.ndarray, bits_O: int, bits_R: int, slot_of_coord) -> np.ndarray:
    """Rows of 128 codes -> bytes[N, 8 (bits_O + bits_R)]: the half-O stream (64 codes of bits_O
    bits, slot s at bits [bits_O s, bits_O s + bits_O)), then the half-R stream."""
    N = idx.shape[0]
    parts = []
    for g, bits in ((0, bits_O), (1, bits_R)):
        part = np.zeros((N, HALF * bits // 8), dtype=np.uint8)
        for j in range(HALF * g, HALF * (g + 1)):
            s = slot_of_coord(j)
            for i in range(bits):
                k = bits * s + i
                part[:, k // 8] |= (((idx[:, j] >> i) & 1).astype(np.uint8)) << (k % 8)
        parts.append(part)
    return np.concatenate(parts, axis=1)


def unpack_codes_mixed(rows: np.ndarray, bits_O: int, bits_R: int, slot_of_coord) -> np.ndarray:
    rows = np.asarray(rows, dtype=np.uint8)
    N = rows.shape[0]
    idx = np.zeros((N, D), dtype=np.int64)
    off = 0
    for g, bits in ((0, bits_O), (1, bits_R)):
        for j in range(HALF * g, HALF * (g + 1)):
            s = slot_of_coord(j)
            for i in range(bits):
                k = bits * s + i
                idx[:, j] |= ((rows[:, off + k // 8] >> (k % 8)) & 1).astype(np.int64) << i
        off += HALF * bits // 8
    return idx


def quantize_cache_mixed(K: np.ndarray, V: np.ndarray, Pi_blk: np.ndarray, outlier_channels,
                         k_bits: tuple, v_bits: tuple, S: Optional[np.ndarray]) -> dict:
    """K, V: [B, Hkv, T, d]; k_bits, v_bits = (bits_O, bits_R).  Packed arrays in the mixed
    layout (norms [B, Hkv, T, 2] = (n_O, n_R)) plus the float64 intermediates."""
    B, H, T, d = K.shape
    kq = quantize_vectors_mixed(K.reshape(-1, d), Pi_blk, outlier_channels, *k_bits, S)
    vq = quantize_vectors_mixed(V.reshape(-1, d), Pi_blk, outlier_channels, *v_bits, None)
    cache = {
        "k_codes": pack_codes_mixed(kq["idx"], *k_bits, k_slot_of_coord_mixed).reshape(B, H, T, -1),
        "k_norm": np.stack([kq["n_O"], kq["n_R"]], -1).astype(np.float32).reshape(B, H, T, 2),
        "v_codes": pack_codes_mixed(vq["idx"], *v_bits, v_slot_of_coord_mixed).reshape(B, H, T, -1),
        "v_norm": np.stack([vq["n_O"], vq["n_R"]], -1).astype(np.float32).reshape(B, H, T, 2),
        "k_u": kq["u"].reshape(B, H, T, d), "k_idx": kq["idx"].reshape(B, H, T, d),
        "v_u": vq["u"].reshape(B, H, T, d), "v_idx": vq["idx"].reshape(B, H, T, d),
    }
    if S is not None:
        cache["k_signs"] = pack_signs(kq["signs"]).reshape(B, H, T, -1)
        cache["k_rnorm"] = kq["rnorm"].astype(np.float32).reshape(B, H, T)
        cache["k_sproj"] = kq["sproj"].reshape(B, H, T, -1)
    return cache


def dequantize_mixed(codes: np.ndarray, norms: np.ndarray, bits: tuple, slot_of_coord) -> np.ndarray:
    """khat (or vhat) in the block-rotated basis: half g = (n_g / sqrt(64)) c_g[idx_g]."""
    idx = unpack_codes_mixed(codes, bits[0], bits[1], slot_of_coord)
    norms = np.asarray(norms, np.float64)
    out = np.zeros(idx.shape, dtype=np.float64)
    for g in range(2):
        cols = slice(HALF * g, HALF * (g + 1))
        out[:, cols] = (norms[:, g:g + 1] / math.sqrt(HALF)) * codebook(bits[g]).centroids[idx[:, cols]]
    return out


def decode_attention_mixed(q: np.ndarray, Pi_blk: np.ndarray, S: Optional[np.ndarray], cache: dict,
                           k_bits: tuple, v_bits: tuple, seq_len: int,
                           scale: Optional[float] = None) -> np.ndarray:
    """Decode attention over a mixed-layout cache: est_i = <q', khat_i> + ||r_i|| sqrt(pi/2)/m
    <S q', 2 sign_i - 1>, q' = Pi_blk q; o = Pi_blk^T sum_i softmax(scale est)_i vhat_i."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = cache["k_codes"].shape[1]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    P = np.asarray(Pi_blk, dtype=np.float64)
    out = np.zeros((B, Hq, d))
    for b in range(B):
        for kv in range(Hkv):
            sl = (b, kv, slice(0, seq_len))
            khat = dequantize_mixed(cache["k_codes"][sl], cache["k_norm"][sl], k_bits, k_slot_of_coord_mixed)
            vhat = dequantize_mixed(cache["v_codes"][sl], cache["v_norm"][sl], v_bits, v_slot_of_coord_mixed)
            for h in range(kv * g, (kv + 1) * g):
                qp = P @ q[b, h]
                est = khat @ qp
                if S is not None:
                    S64 = np.asarray(S, np.float64)
                    pm = 2.0 * unpack_signs(cache["k_signs"][sl]) - 1.0
                    est = est + np.asarray(cache["k_rnorm"][sl], np.float64) * (SQRT_PI_OVER_2 / S64.shape[0]) * (pm @ (S64 @ qp))
                out[b, h] = P.T @ softmax_weighted_sum(scale * est, vhat)
    return out


def code_exempt_mixed(u: np.ndarray, bits_O: int, bits_R: int, band: float = 1e-6) -> np.ndarray:
    """Per coordinate: within `band` of a threshold of its half's codebook."""
    ex = np.zeros(u.shape, dtype=bool)
    for g, bits in ((0, bits_O), (1, bits_R)):
        cols = slice(HALF * g, HALF * (g + 1))
        ex[..., cols] = code_exempt(u[..., cols], bits, band)
    return ex


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
    "HALF", "quantize_vectors_mixed", "k_slot_of_coord_mixed", "v_slot_of_coord_mixed",
    "pack_codes_mixed", "unpack_codes_mixed", "quantize_cache_mixed", "dequantize_mixed",
    "decode_attention_mixed", "code_exempt_mixed",
]
