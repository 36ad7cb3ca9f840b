"""Seeded synthetic inputs for compressed-KV attention (shared by the oracle, tests and bench).

This module draws random numbers and nothing else: it holds none of the
quantizer's arithmetic (no codebook, no rotation of data, no packing, no
attention).  The random objects the method itself draws -- the orthogonal
rotation Pi and the QJL sketch matrix S -- are produced here as plain inputs,
so that the CPU oracle and the CUDA path receive identical matrices.

Workload recipes follow the five configurations of the method's scope table
(the shapes the pages benchmark: a single head with outlier channels, a
Llama-3-8B-shaped layer at 32K and 128K context, a Llama-3-70B-shaped layer,
and a 1M-token MoE-style layer).  The pages measure real models (wikitext-2,
LongBench, Needle); none is available, so these seeded Gaussians stand in:

* K and V entries are N(0,1) times a per-(kv-head, channel) scale
  exp(sigma * z), z ~ N(0,1);
* "outlier channels": round(frac * head_dim) channels per kv-head (chosen by
  a seeded permutation) whose scale is multiplied by a factor;
* "heavy tail": each entry is replaced, with probability p, by a Student-t(3)
  draw Z / sqrt(chi2_3 / 3) built from four normals;
* bf16 inputs are rounded to nearest even from fp32; fp32 inputs stay fp32;
* queries are N(0,1) fp32.

Every tensor is drawn with a torch.Generator seeded from the config's seed s
with fixed sub-streams (K: 10s+1, V: 10s+2, q: 10s+3, scales: 10s+4,
outlier choice: 10s+5, heavy-tail mask and draws: 10s+6/10s+7).  Pi uses seed
1000+s, S uses 2000+s.  Values depend on the device the generator runs on
(torch's CPU and CUDA generators differ); callers that compare two
implementations always hand both the same tensors.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

HEAD_DIM = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention layer's worth of KV-cache work."""

    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    T: int
    k_bits: int
    v_bits: int
    qjl_m: int
    in_dtype: str  # "fp32" | "bf16"
    sigma: float  # lognormal sigma of per-channel scales (0 = no scales)
    outlier_channels: int  # per kv-head
    outlier_factor: float
    t3_prob: float  # probability an entry is Student-t(3)
    chunk: int  # streaming-quantize chunk length (tokens); T = one chunk
    head_dim: int = HEAD_DIM
    rotation: str = "haar"  # "haar" (dense Haar-random) | "hadamard" (D1 H D2 H D3 / d)
    layout: str = "plain"   # "plain" | "mixed" (outlier half at k_bits / v_bits, the rest one bit fewer)

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def scaled(self, T: Optional[int] = None, B: Optional[int] = None,
               Hkv: Optional[int] = None, Hq: Optional[int] = None,
               chunk: Optional[int] = None, name: Optional[str] = None) -> "Workload":
        """Same recipe at a smaller size (for tests the CPU oracle finishes)."""
        T2 = T if T is not None else self.T
        return dataclasses.replace(
            self,
            name=name or f"{self.name}@T{T2}",
            T=T2,
            B=B if B is not None else self.B,
            Hkv=Hkv if Hkv is not None else self.Hkv,
            Hq=Hq if Hq is not None else self.Hq,
            chunk=min(chunk if chunk is not None else self.chunk, T2) if T2 > 0 else 0,
        )

    # compressed bytes per token per kv-head (codes + signs + norms)
    def _code_bytes(self, bits: int) -> int:
        return 8 * (2 * bits - 1) if self.layout == "mixed" else 16 * bits

    def k_row_bytes(self) -> int:
        nb = 8 if self.layout == "mixed" else 4
        return self._code_bytes(self.k_bits) + (16 + 4 if self.qjl_m else 0) + nb

    def v_row_bytes(self) -> int:
        return self._code_bytes(self.v_bits) + (8 if self.layout == "mixed" else 4)

    def decode_bytes(self, seq_len: Optional[int] = None) -> int:
        T = self.T if seq_len is None else seq_len
        return self.B * self.Hkv * T * (self.k_row_bytes() + self.v_row_bytes())

    def quantize_bytes(self, tokens: Optional[int] = None) -> int:
        T = self.T if tokens is None else tokens
        elt = 4 if self.in_dtype == "fp32" else 2
        return self.B * self.Hkv * T * (2 * self.head_dim * elt
                                        + self.k_row_bytes() + self.v_row_bytes())


# The five configurations (seed 0 is given for the single-head case; the
# others take seeds 1..4 in order).
CONFIGS = {
    "single_head_4k": Workload("single_head_4k", 0, B=1, Hq=16, Hkv=1, T=4096,
                               k_bits=3, v_bits=3, qjl_m=128, in_dtype="fp32",
                               sigma=0.0, outlier_channels=4, outlier_factor=20.0,
                               t3_prob=0.0, chunk=4096),
    "llama3_8b_32k": Workload("llama3_8b_32k", 1, B=1, Hq=32, Hkv=8, T=32768,
                              k_bits=3, v_bits=3, qjl_m=128, in_dtype="bf16",
                              sigma=0.5, outlier_channels=3, outlier_factor=15.0,
                              t3_prob=0.0, chunk=32768),
    "llama3_8b_128k_b4": Workload("llama3_8b_128k_b4", 2, B=4, Hq=32, Hkv=8, T=131072,
                                  k_bits=4, v_bits=4, qjl_m=128, in_dtype="bf16",
                                  sigma=0.5, outlier_channels=3, outlier_factor=15.0,
                                  t3_prob=0.0, chunk=131072),
    "llama3_70b_16k_b16": Workload("llama3_70b_16k_b16", 3, B=16, Hq=64, Hkv=8, T=16384,
                                   k_bits=3, v_bits=2, qjl_m=128, in_dtype="bf16",
                                   sigma=0.7, outlier_channels=0, outlier_factor=1.0,
                                   t3_prob=0.01, chunk=16384),
    "moe_1m": Workload("moe_1m", 4, B=1, Hq=16, Hkv=2, T=1048576,
                       k_bits=4, v_bits=4, qjl_m=128, in_dtype="bf16",
                       sigma=0.5, outlier_channels=3, outlier_factor=15.0,
                       t3_prob=0.0, chunk=8192),
}
CONFIG_ORDER = ["single_head_4k", "llama3_8b_32k", "llama3_8b_128k_b4",
                "llama3_70b_16k_b16", "moe_1m"]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_rotation(seed: int, d: int = HEAD_DIM) -> np.ndarray:
    """Haar-random orthogonal d x d matrix, rounded to fp32.

    G ~ N(0,1)^{d x d} in float64 (CPU generator, seed 1000+s by convention),
    G = QR, columns of Q multiplied by sign(R_jj) so the draw is Haar.
    """
    g = _gen(seed, "cpu")
    G = torch.randn(d, d, dtype=torch.float64, generator=g)
    Q, R = torch.linalg.qr(G)
    Q = Q * torch.sign(torch.diagonal(R)).unsqueeze(0)
    return Q.to(torch.float32).numpy().copy()


def make_qjl_matrix(seed: int, m: int = 128, d: int = HEAD_DIM) -> np.ndarray:
    """Gaussian m x d sketch matrix with entries rounded to the nearest fp16 (stored fp32)."""
    g = _gen(seed, "cpu")
    S = torch.randn(m, d, dtype=torch.float64, generator=g)
    return S.to(torch.float16).to(torch.float32).numpy().copy()


_U64 = (1 << 64) - 1


def splitmix64(seed: int, n: int) -> int:
    """Output n (0, 1, ...) of the SplitMix64 generator started at state `seed` (Steele, Lea and
    Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014): the state advances by
    0x9E3779B97F4A7C15 and each output is the state after two xor-shift-multiply rounds."""
    z = (int(seed) + (int(n) + 1) * 0x9E3779B97F4A7C15) & _U64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _U64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _U64
    return z ^ (z >> 31)


def make_hadamard_rotation(seed: int, d: int = HEAD_DIM) -> np.ndarray:
    """Structured orthogonal d x d matrix D1 H D2 H D3 / d (fp32, every entry a multiple of 2/d).

    H is the Sylvester Hadamard matrix (H[i][j] = (-1)^popcount(i & j)); D_k = diag(s_k) with
    s_k[i] = +1 if SplitMix64 output k*d + i of `seed` is even, else -1.
    """
    assert d & (d - 1) == 0
    idx = np.arange(d)
    H = np.array([[(-1) ** bin(i & j).count("1") for j in idx] for i in idx], dtype=np.float64)
    s = np.array([[1.0 if splitmix64(seed, k * d + i) % 2 == 0 else -1.0 for i in idx] for k in range(3)])
    P = (s[0][:, None] * H) @ (s[1][:, None] * H) * s[2][None, :] / d
    return P.astype(np.float32)


def make_block_rotation(seed: int, outlier_channels, d: int = HEAD_DIM) -> np.ndarray:
    """Rotation of the outlier-aware mixed-precision layout: two independent Haar-random
    (d/2) x (d/2) matrices (seeds `seed` and `seed` + 1, drawn like make_rotation), the first
    acting on the outlier channels (ascending) into rows 0 .. d/2 - 1, the second on the other
    channels into rows d/2 .. d - 1.  fp32."""
    half = d // 2
    O = np.sort(np.asarray(outlier_channels, dtype=np.int64))
    assert O.size == half and np.unique(O).size == half and O.min() >= 0 and O.max() < d
    R = np.setdiff1d(np.arange(d), O)
    P = np.zeros((d, d), dtype=np.float32)
    P[:half][:, O] = make_rotation(seed, half)
    P[half:][:, R] = make_rotation(seed + 1, half)
    return P


def outlier_channels_for(w: Workload, count: int = HEAD_DIM // 2) -> np.ndarray:
    """The `count` channels with the largest key scale summed over the kv-heads, from the
    workload's own per-channel scale draw (a per-layer choice, as the outlier-aware variant keeps
    one channel split per layer); ascending channel indices."""
    sc = _channel_scales(w, 0, "cpu").sum(dim=0)
    order = torch.argsort(sc, descending=True, stable=True)[:count]
    return np.sort(order.numpy().astype(np.int64))


def rotation_for(w: Workload) -> np.ndarray:
    if w.layout == "mixed":
        return make_block_rotation(1000 + w.seed, outlier_channels_for(w), w.head_dim)
    if w.rotation == "hadamard":
        return make_hadamard_rotation(1000 + w.seed, w.head_dim)
    assert w.rotation == "haar", w.rotation
    return make_rotation(1000 + w.seed, w.head_dim)


def qjl_for(w: Workload) -> Optional[np.ndarray]:
    return make_qjl_matrix(2000 + w.seed, w.qjl_m, w.head_dim) if w.qjl_m else None


def _channel_scales(w: Workload, which: int, device) -> torch.Tensor:
    """Per-(kv-head, channel) multiplicative scales, shape [Hkv, d], fp32."""
    d = w.head_dim
    scales = torch.ones(w.Hkv, d, dtype=torch.float32, device=device)
    if w.sigma > 0:
        g = _gen(10 * w.seed + 4, device)
        z = torch.randn(2, w.Hkv, d, dtype=torch.float32, device=device, generator=g)[which]
        scales = torch.exp(w.sigma * z)
    if w.outlier_channels > 0:
        g = _gen(10 * w.seed + 5, device)
        for which_i in range(2):
            for h in range(w.Hkv):
                perm = torch.randperm(d, generator=g, device=device)[: w.outlier_channels]
                if which_i == which:
                    scales[h, perm] *= w.outlier_factor
    return scales


def make_kv(w: Workload, which: str, device="cpu", T: Optional[int] = None,
            t_start: int = 0) -> torch.Tensor:
    """K (which='k') or V (which='v') as [B, Hkv, T, d] in the workload's input dtype.

    ``t_start``/``T`` select a token window of the full draw only in the sense
    of shape; every call draws the whole [B, Hkv, T, d] block from its seed.
    """
    assert which in ("k", "v")
    idx = 0 if which == "k" else 1
    T = w.T if T is None else T
    shape = (w.B, w.Hkv, T, w.head_dim)
    g = _gen(10 * w.seed + 1 + idx, device)
    x = torch.randn(shape, dtype=torch.float32, device=device, generator=g)
    if w.t3_prob > 0:
        gm = _gen(10 * w.seed + 6 + 2 * idx, device)
        mask = torch.rand(shape, dtype=torch.float32, device=device, generator=gm) < w.t3_prob
        gt = _gen(10 * w.seed + 7 + 2 * idx, device)
        zc = torch.randn((4,) + shape, dtype=torch.float32, device=device, generator=gt)
        chi2 = zc[1] * zc[1] + zc[2] * zc[2] + zc[3] * zc[3]
        t3 = zc[0] / torch.sqrt(chi2 / 3.0)
        x = torch.where(mask, t3, x)
        del zc, chi2, t3, mask
    x.mul_(_channel_scales(w, idx, device).view(1, w.Hkv, 1, w.head_dim))
    if w.in_dtype == "bf16":
        return x.to(torch.bfloat16)
    return x


def make_queries(w: Workload, device="cpu") -> torch.Tensor:
    """Decode queries q ~ N(0,1), shape [B, Hq, d], fp32."""
    g = _gen(10 * w.seed + 3, device)
    return torch.randn((w.B, w.Hq, w.head_dim), dtype=torch.float32, device=device, generator=g)


def gqa_kv_head(h: int, Hq: int, Hkv: int) -> int:
    """Query head h reads kv-head h // (Hq / Hkv)."""
    return h // (Hq // Hkv)


def shard_units(n_units: int, rank: int, world: int) -> range:
    """Contiguous block of independent (batch, kv-head) units owned by one rank."""
    per = n_units // world
    extra = n_units % world
    start = rank * per + min(rank, extra)
    stop = start + per + (1 if rank < extra else 0)
    return range(start, stop)


def nbytes_human(n: int) -> str:
    for unit in ("B", "KB", "MB", "GB"):
        if n < 1024:
            return f"{n:.1f} {unit}"
        n /= 1024
    return f"{n:.1f} TB"


__all__ = [
    "HEAD_DIM", "Workload", "CONFIGS", "CONFIG_ORDER", "make_rotation", "make_hadamard_rotation",
    "make_block_rotation", "outlier_channels_for",
    "splitmix64", "make_qjl_matrix",
    "rotation_for", "qjl_for", "make_kv", "make_queries", "gqa_kv_head", "shard_units",
    "nbytes_human",
]
