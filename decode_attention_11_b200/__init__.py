"""B200-native TurboQuant-style compressed-KV hot path: Python binding of the tq C ABI.

Argument marshalling only: every step of the path runs in ``libtq_b200.so`` (CUDA kernels for
sm_100a plus the host codebook builder).  PyTorch provides device memory and streams.  There is
no fallback: if the shared library is missing or fails to load, every call raises.

    import decode_attention_11_b200 as tq
    params = tq.Params.create(Pi, S, k_bits=4, v_bits=4, device="cuda")
    cache = tq.Cache.allocate(B, Hkv, T_cap, k_bits=4, v_bits=4, qjl_m=128, device="cuda")
    tq.quantize(params, k, v, cache, t_offset=0)            # k, v: [B, Hkv, T_new, 128]
    out = tq.decode_attn(params, q, cache, seq_len)          # q: [B, Hq, 128]
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# TQ_DEBUG=1 selects the build with the decode kernel's device-side bounds checks
# (python -m decode_attention_11_b200.build --debug)
LIB_PATH = os.path.join(_HERE, "libtq_b200_debug.so" if os.environ.get("TQ_DEBUG") == "1"
                        else "libtq_b200.so")

TQ_OK = 0
TQ_ERR_INVALID_ARG = 1
TQ_ERR_UNSUPPORTED = 2
TQ_ERR_NO_CONVERGENCE = 3
TQ_ERR_WORKSPACE = 4
TQ_ERR_CUDA = 5
TQ_F32 = 0
TQ_BF16 = 1
TQ_LAYOUT_PLAIN = 0
TQ_LAYOUT_MIXED = 1

# Functions declared in include/tq.h (checked by the test-suite against the header).
EXPORTED = ("tq_status_string", "tq_last_error", "tq_version", "tq_build_codebook",
            "tq_quantize", "tq_quantize_device_errors", "tq_quantize_vector_fixups",
            "tq_quantize_code_fixups", "tq_quantize_exempt_codes", "tq_quantize_exempt_signs",
            "tq_decode_workspace_size", "tq_decode_attn", "tq_decode_attn_static",
            "tq_decode_static_workspace_limit", "tq_sketch_rotation", "tq_build_hadamard_rotation",
            "tq_decode_step", "tq_decode_step_fused", "tq_decode_device_errors",
            "tq_reset_device_errors", "tq_debug_quantize_stall")


class TqError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{status_string(status)}: {detail}")
        self.status = status


class _Cache(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hkv", ctypes.c_int), ("T_cap", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("k_bits", ctypes.c_int), ("v_bits", ctypes.c_int),
                ("qjl_m", ctypes.c_int),
                ("k_codes", ctypes.c_void_p), ("k_signs", ctypes.c_void_p),
                ("k_norm", ctypes.c_void_p), ("k_rnorm", ctypes.c_void_p),
                ("v_codes", ctypes.c_void_p), ("v_norm", ctypes.c_void_p),
                ("layout", ctypes.c_int)]


class _Params(ctypes.Structure):
    _fields_ = [("Pi", ctypes.c_void_p), ("S", ctypes.c_void_p),
                ("k_centroids", ctypes.c_void_p), ("k_thresholds", ctypes.c_void_p),
                ("v_centroids", ctypes.c_void_p), ("v_thresholds", ctypes.c_void_p),
                ("S_Pi", ctypes.c_void_p),
                ("k_centroids_lo", ctypes.c_void_p), ("k_thresholds_lo", ctypes.c_void_p),
                ("v_centroids_lo", ctypes.c_void_p), ("v_thresholds_lo", ctypes.c_void_p),
                ("outlier_mask", ctypes.c_uint32 * 4)]


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libtq_b200.so, or libtq_b200_debug.so under TQ_DEBUG=1 (raises if it is missing:
    there is no other implementation)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} not built; run `python -m decode_attention_11_b200.build`"
                           + (" --debug" if LIB_PATH.endswith("_debug.so") else ""))
    L = ctypes.CDLL(LIB_PATH)
    L.tq_status_string.restype = ctypes.c_char_p
    L.tq_status_string.argtypes = [ctypes.c_int]
    L.tq_last_error.restype = ctypes.c_char_p
    L.tq_last_error.argtypes = []
    L.tq_version.restype = ctypes.c_int
    L.tq_build_codebook.restype = ctypes.c_int
    L.tq_build_codebook.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                    ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float),
                                    ctypes.POINTER(ctypes.c_double)]
    L.tq_quantize.restype = ctypes.c_int
    L.tq_quantize.argtypes = [ctypes.POINTER(_Params), ctypes.c_void_p, ctypes.c_void_p,
                              ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                              ctypes.c_int, ctypes.c_int, ctypes.POINTER(_Cache), ctypes.c_void_p]
    L.tq_quantize_device_errors.restype = ctypes.c_int
    L.tq_quantize_device_errors.argtypes = []
    L.tq_quantize_vector_fixups.restype = ctypes.c_longlong
    L.tq_quantize_vector_fixups.argtypes = []
    L.tq_quantize_code_fixups.restype = ctypes.c_longlong
    L.tq_quantize_code_fixups.argtypes = []
    L.tq_quantize_exempt_codes.restype = ctypes.c_longlong
    L.tq_quantize_exempt_codes.argtypes = []
    L.tq_quantize_exempt_signs.restype = ctypes.c_longlong
    L.tq_quantize_exempt_signs.argtypes = []
    L.tq_reset_device_errors.restype = ctypes.c_int
    L.tq_reset_device_errors.argtypes = []
    L.tq_debug_quantize_stall.restype = ctypes.c_int
    L.tq_debug_quantize_stall.argtypes = [ctypes.c_int, ctypes.c_longlong]
    L.tq_decode_device_errors.restype = ctypes.c_int
    L.tq_decode_device_errors.argtypes = []
    L.tq_decode_step_fused.restype = ctypes.c_int
    L.tq_decode_step_fused.argtypes = [ctypes.POINTER(_Cache), ctypes.c_int, ctypes.c_int]
    L.tq_decode_workspace_size.restype = ctypes.c_size_t
    L.tq_decode_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(_Cache),
                                           ctypes.c_int]
    L.tq_decode_attn.restype = ctypes.c_int
    L.tq_decode_attn.argtypes = [ctypes.POINTER(_Params), ctypes.c_void_p, ctypes.c_int,
                                 ctypes.c_int, ctypes.POINTER(_Cache), ctypes.c_int, ctypes.c_float,
                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    L.tq_decode_attn_static.restype = ctypes.c_int
    L.tq_decode_attn_static.argtypes = [ctypes.POINTER(_Params), ctypes.c_void_p, ctypes.c_int,
                                        ctypes.c_int, ctypes.POINTER(_Cache), ctypes.c_int,
                                        ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
    L.tq_decode_static_workspace_limit.restype = ctypes.c_size_t
    L.tq_decode_static_workspace_limit.argtypes = []
    L.tq_decode_step.restype = ctypes.c_int
    L.tq_decode_step.argtypes = [ctypes.POINTER(_Params), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                 ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.POINTER(_Cache),
                                 ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                 ctypes.c_size_t, ctypes.c_void_p]
    L.tq_build_hadamard_rotation.restype = ctypes.c_int
    L.tq_build_hadamard_rotation.argtypes = [ctypes.c_uint64, ctypes.POINTER(ctypes.c_float)]
    L.tq_sketch_rotation.restype = ctypes.c_int
    L.tq_sketch_rotation.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                     ctypes.c_void_p]
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().tq_status_string(int(status)).decode()


def last_error() -> str:
    return lib().tq_last_error().decode()


def _check(status: int) -> None:
    if status != TQ_OK:
        raise TqError(status, last_error())


def version() -> int:
    return int(lib().tq_version())


def build_codebook(bits: int, max_iter: int = 100000, tol: float = 1e-13
                   ) -> Tuple[np.ndarray, np.ndarray, float]:
    """Lloyd-Max quantizer of N(0,1): (centroids float32[2^b], thresholds float32[2^b-1], distortion)."""
    L = 1 << bits if 1 <= bits <= 8 else 1
    c = np.zeros(max(L, 1), dtype=np.float32)
    t = np.zeros(max(L - 1, 1), dtype=np.float32)
    dist = ctypes.c_double(0.0)
    _check(lib().tq_build_codebook(int(bits), int(max_iter), float(tol),
                                   c.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                   t.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                   ctypes.byref(dist)))
    return c[:L], t[:L - 1], float(dist.value)


def build_hadamard_rotation(seed: int) -> np.ndarray:
    """Structured orthogonal rotation D1 H D2 H D3 / 128 (tq_build_hadamard_rotation), fp32 [128, 128]."""
    P = np.empty((128, 128), dtype=np.float32)
    _check(lib().tq_build_hadamard_rotation(int(seed) & ((1 << 64) - 1),
                                            P.ctypes.data_as(ctypes.POINTER(ctypes.c_float))))
    return P


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if stream.cuda_stream else None


def sketch_rotation_product(Pi: torch.Tensor, S: torch.Tensor, stream=None) -> torch.Tensor:
    """S Pi in fp64 on the device of Pi (tq_sketch_rotation), for Params.S_Pi."""
    if not (Pi.is_cuda and S.is_cuda and Pi.device == S.device):
        raise ValueError("Pi and S must be on the same CUDA device")
    if Pi.dtype != torch.float32 or S.dtype != torch.float32 or tuple(Pi.shape) != (128, 128) \
            or S.dim() != 2 or S.shape[1] != 128:
        raise ValueError("Pi must be fp32 [128, 128] and S fp32 [m, 128]")
    Pi = Pi.contiguous()
    S = S.contiguous()
    out = torch.empty(S.shape[0], 128, dtype=torch.float64, device=Pi.device)
    with torch.cuda.device(Pi.device):
        _check(lib().tq_sketch_rotation(Pi.data_ptr(), S.data_ptr(), int(S.shape[0]), out.data_ptr(),
                                        _stream_ptr(stream)))
    return out


@dataclasses.dataclass
class Params:
    """Per-layer constants on the device (fp32): rotation, sketch, codebooks."""

    Pi: torch.Tensor
    S: Optional[torch.Tensor]
    k_centroids: torch.Tensor
    k_thresholds: torch.Tensor
    v_centroids: torch.Tensor
    v_thresholds: torch.Tensor
    S_Pi: Optional[torch.Tensor] = None
    # mixed layout: codebooks of the non-outlier half (one bit fewer) and the outlier channels
    k_centroids_lo: Optional[torch.Tensor] = None
    k_thresholds_lo: Optional[torch.Tensor] = None
    v_centroids_lo: Optional[torch.Tensor] = None
    v_thresholds_lo: Optional[torch.Tensor] = None
    outlier_mask: tuple = (0, 0, 0, 0)

    @classmethod
    def create(cls, Pi, S, k_bits: int, v_bits: int, device="cuda", sketch_rotation=True,
               outlier_channels=None) -> "Params":
        """Upload the constants; with a sketch, also S Pi in fp64 (tq_sketch_rotation) unless
        `sketch_rotation` is False.  With `outlier_channels` (64 channel indices) the constants
        are those of the mixed layout: Pi must then be the block rotation of those channels."""
        kc, kt, _ = build_codebook(k_bits)
        vc, vt, _ = build_codebook(v_bits)
        f = lambda x: torch.as_tensor(np.ascontiguousarray(x, dtype=np.float32)).to(device)
        p = cls(f(Pi), None if S is None else f(S), f(kc), f(kt), f(vc), f(vt))
        if outlier_channels is not None:
            kc2, kt2, _ = build_codebook(k_bits - 1)
            vc2, vt2, _ = build_codebook(v_bits - 1)
            p.k_centroids_lo, p.k_thresholds_lo = f(kc2), f(kt2)
            p.v_centroids_lo, p.v_thresholds_lo = f(vc2), f(vt2)
            mask = [0, 0, 0, 0]
            for c in np.asarray(outlier_channels, dtype=np.int64).tolist():
                mask[c // 32] |= 1 << (c % 32)
            p.outlier_mask = tuple(mask)
        if p.S is not None and sketch_rotation and p.Pi.is_cuda:
            p.S_Pi = sketch_rotation_product(p.Pi, p.S)
        return p

    def as_c(self) -> _Params:
        return _Params(_ptr(self.Pi), _ptr(self.S), _ptr(self.k_centroids),
                       _ptr(self.k_thresholds), _ptr(self.v_centroids), _ptr(self.v_thresholds),
                       _ptr(self.S_Pi), _ptr(self.k_centroids_lo), _ptr(self.k_thresholds_lo),
                       _ptr(self.v_centroids_lo), _ptr(self.v_thresholds_lo),
                       (ctypes.c_uint32 * 4)(*self.outlier_mask))


@dataclasses.dataclass
class Cache:
    """Packed cache arrays (caller-owned torch tensors; layout in include/tq.h)."""

    B: int
    Hkv: int
    T_cap: int
    k_bits: int
    v_bits: int
    qjl_m: int
    k_codes: torch.Tensor
    k_signs: Optional[torch.Tensor]
    k_norm: torch.Tensor
    k_rnorm: Optional[torch.Tensor]
    v_codes: torch.Tensor
    v_norm: torch.Tensor
    layout: int = TQ_LAYOUT_PLAIN

    @staticmethod
    def code_bytes(bits: int, layout: int) -> int:
        """Bytes of a packed row of 128 codes (mixed layout: halves of bits and bits - 1)."""
        return 8 * (2 * bits - 1) if layout == TQ_LAYOUT_MIXED else 16 * bits

    @classmethod
    def allocate(cls, B, Hkv, T_cap, k_bits, v_bits, qjl_m=128, device="cuda",
                 layout=TQ_LAYOUT_PLAIN) -> "Cache":
        u8 = dict(dtype=torch.uint8, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        nrm = (2,) if layout == TQ_LAYOUT_MIXED else ()
        return cls(B, Hkv, T_cap, k_bits, v_bits, qjl_m,
                   torch.zeros(B, Hkv, T_cap, cls.code_bytes(k_bits, layout), **u8),
                   torch.zeros(B, Hkv, T_cap, 16, **u8) if qjl_m else None,
                   torch.zeros(B, Hkv, T_cap, *nrm, **f32),
                   torch.zeros(B, Hkv, T_cap, **f32) if qjl_m else None,
                   torch.zeros(B, Hkv, T_cap, cls.code_bytes(v_bits, layout), **u8),
                   torch.zeros(B, Hkv, T_cap, *nrm, **f32), layout)

    @classmethod
    def from_arrays(cls, arrays: dict, k_bits, v_bits, qjl_m, device="cuda",
                    layout=TQ_LAYOUT_PLAIN) -> "Cache":
        """Wrap host arrays (k_codes, k_signs, k_norm, k_rnorm, v_codes, v_norm) as a device cache."""
        g = lambda n: None if arrays.get(n) is None else torch.as_tensor(
            np.ascontiguousarray(arrays[n])).to(device)
        kc = g("k_codes")
        B, Hkv, T_cap = kc.shape[:3]
        return cls(B, Hkv, T_cap, k_bits, v_bits, qjl_m, kc, g("k_signs") if qjl_m else None,
                   g("k_norm"), g("k_rnorm") if qjl_m else None, g("v_codes"), g("v_norm"), layout)

    def as_c(self) -> _Cache:
        return _Cache(self.B, self.Hkv, self.T_cap, 128, self.k_bits, self.v_bits, self.qjl_m,
                      _ptr(self.k_codes), _ptr(self.k_signs), _ptr(self.k_norm),
                      _ptr(self.k_rnorm), _ptr(self.v_codes), _ptr(self.v_norm), self.layout)

    def row_bytes(self) -> int:
        nb = 8 if self.layout == TQ_LAYOUT_MIXED else 4
        return (self.code_bytes(self.k_bits, self.layout) + (20 if self.qjl_m else 0) + nb
                + self.code_bytes(self.v_bits, self.layout) + nb)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TQ_F32
    if t.dtype == torch.bfloat16:
        return TQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def quantize(params: Params, k: torch.Tensor, v: torch.Tensor, cache: Cache, t_offset: int = 0,
             stream=None) -> None:
    """Compress k, v ([B, Hkv, T_new, 128], same strides, last dim contiguous) into cache rows
    [t_offset, t_offset + T_new)."""
    if k.shape != v.shape or k.stride() != v.stride() or k.dtype != v.dtype:
        raise ValueError("k and v must share shape, strides and dtype")
    if k.dim() != 4 or k.shape[-1] != 128 or k.stride(-1) != 1:
        raise ValueError("k must be [B, Hkv, T_new, 128] with a contiguous last dim")
    c = cache.as_c()
    p = params.as_c()
    _check(lib().tq_quantize(ctypes.byref(p), k.data_ptr(), v.data_ptr(), _dtype_code(k),
                             k.stride(0), k.stride(1), k.stride(2), k.shape[2], int(t_offset),
                             ctypes.byref(c), _stream_ptr(stream)))


def quantize_device_errors() -> int:
    """Device-side error bits recorded by tq_quantize (0 = none); synchronizes."""
    return int(lib().tq_quantize_device_errors())


def quantize_vector_fixups() -> int:
    """Key vectors re-derived in fp64 by tq_quantize so far (diagnostic); synchronizes."""
    return int(lib().tq_quantize_vector_fixups())


def quantize_code_fixups() -> int:
    """Coordinates re-derived in fp64 by tq_quantize so far (diagnostic); synchronizes."""
    return int(lib().tq_quantize_code_fixups())


def quantize_exempt_codes() -> int:
    """Coordinates so far whose exact rotated value lay within 1e-6 of a threshold (the cases the
    parity rule exempts; divide by 256 per quantized (token, kv-head) for the fraction)."""
    return int(lib().tq_quantize_exempt_codes())


def quantize_exempt_signs() -> int:
    """QJL sketch values so far that were flagged near 0 and lay within 1e-5 of 0 exactly."""
    return int(lib().tq_quantize_exempt_signs())


def reset_device_errors() -> None:
    """Clear the recorded device error bits of both operations; synchronizes."""
    if lib().tq_reset_device_errors() != 0:
        raise TqError(TQ_ERR_CUDA, "could not reach the device")


def debug_quantize_stall(enable: bool, wait_cycles: int = 0) -> None:
    """Test hook: make the bf16 quantize kernel's bounded waits run out (see tq.h)."""
    _check(lib().tq_debug_quantize_stall(1 if enable else 0, int(wait_cycles)))


def decode_device_errors() -> int:
    """Device-side error bits recorded by tq_decode_attn (0 = none); synchronizes."""
    return int(lib().tq_decode_device_errors())


def decode_step_fused(cache: Cache, Hq: int, t: int) -> bool:
    """Whether decode_step at row t runs as one fused decode launch (see tq_decode_step_fused)."""
    c = cache.as_c()
    r = int(lib().tq_decode_step_fused(ctypes.byref(c), Hq, t))
    if r < 0:
        raise ValueError(f"invalid sizes Hq={Hq} t={t}")
    return r == 1


def decode_workspace_size(B: int, Hq: int, cache: Cache, seq_len: int) -> int:
    c = cache.as_c()
    return int(lib().tq_decode_workspace_size(int(B), int(Hq), ctypes.byref(c), int(seq_len)))


def decode_attn(params: Params, q: torch.Tensor, cache: Cache, seq_len: int,
                out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                scale: float = 0.0, stream=None) -> torch.Tensor:
    """Decode attention of q [B, Hq, 128] over the first seq_len cached tokens -> fp32 [B, Hq, 128]."""
    if q.dim() != 3 or q.shape[-1] != 128 or not q.is_contiguous():
        raise ValueError("q must be a contiguous [B, Hq, 128] tensor")
    B, Hq, _ = q.shape
    if out is None:
        out = torch.empty(B, Hq, 128, dtype=torch.float32, device=q.device)
    need = decode_workspace_size(B, Hq, cache, seq_len)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    c = cache.as_c()
    p = params.as_c()
    _check(lib().tq_decode_attn(ctypes.byref(p), q.data_ptr(), _dtype_code(q), int(Hq),
                                ctypes.byref(c), int(seq_len), float(scale), out.data_ptr(),
                                workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                _stream_ptr(stream)))
    return out


def decode_step(params: Params, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor, cache: Cache,
                t: int, out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                scale: float = 0.0, stream=None) -> torch.Tensor:
    """One decode step: k_new, v_new [B, Hkv, 128] go to cache row t, then q [B, Hq, 128] attends
    over rows [0, t] -> fp32 [B, Hq, 128] (tq_decode_step)."""
    for x, n in ((k_new, "k_new"), (v_new, "v_new"), (q, "q")):
        if x.dim() != 3 or x.shape[-1] != 128 or not x.is_contiguous():
            raise ValueError(f"{n} must be a contiguous [B, H, 128] tensor")
    if k_new.shape != v_new.shape or k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must have the same shape and dtype")
    if tuple(k_new.shape[:2]) != (cache.B, cache.Hkv):
        raise ValueError("k_new must be [B, Hkv, 128] of the cache")
    B, Hq, _ = q.shape
    if out is None:
        out = torch.empty(B, Hq, 128, dtype=torch.float32, device=q.device)
    need = decode_workspace_size(B, Hq, cache, t + 1)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    c = cache.as_c()
    p = params.as_c()
    _check(lib().tq_decode_step(ctypes.byref(p), k_new.data_ptr(), v_new.data_ptr(), _dtype_code(k_new),
                                q.data_ptr(), _dtype_code(q), int(Hq), ctypes.byref(c), int(t), float(scale),
                                out.data_ptr(), workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), _stream_ptr(stream)))
    return out


def decode_static_workspace_limit() -> int:
    """Bytes of the fixed device scratch array behind decode_attn_static."""
    return int(lib().tq_decode_static_workspace_limit())


def decode_attn_static(params: Params, q: torch.Tensor, cache: Cache, seq_len: int,
                       out: Optional[torch.Tensor] = None, scale: float = 0.0,
                       stream=None) -> torch.Tensor:
    """decode_attn for callers that cannot allocate device memory when they run decode (inside
    an allocator callback, under a fixed-footprint runtime, in a plug-in host): the scratch lives
    in a fixed device array inside the library.  Pass `out` to avoid the one allocation this
    wrapper would otherwise make.  Calls that overlap on the device share that array and race."""
    if q.dim() != 3 or q.shape[-1] != 128 or not q.is_contiguous():
        raise ValueError("q must be a contiguous [B, Hq, 128] tensor")
    B, Hq, _ = q.shape
    if out is None:
        out = torch.empty(B, Hq, 128, dtype=torch.float32, device=q.device)
    c = cache.as_c()
    p = params.as_c()
    _check(lib().tq_decode_attn_static(ctypes.byref(p), q.data_ptr(), _dtype_code(q), int(Hq),
                                       ctypes.byref(c), int(seq_len), float(scale), out.data_ptr(),
                                       _stream_ptr(stream)))
    return out


__all__ = [
    "LIB_PATH", "EXPORTED", "TqError", "lib", "status_string", "last_error", "version",
    "build_codebook", "Params", "Cache", "quantize", "quantize_device_errors",
    "decode_attn_static", "decode_static_workspace_limit",
    "quantize_vector_fixups", "quantize_code_fixups", "quantize_exempt_codes", "quantize_exempt_signs",
    "decode_workspace_size", "decode_attn", "decode_device_errors", "reset_device_errors",
    "debug_quantize_stall", "decode_step", "decode_step_fused",
    "TQ_OK", "TQ_ERR_INVALID_ARG", "TQ_ERR_UNSUPPORTED", "TQ_ERR_NO_CONVERGENCE",
    "TQ_ERR_WORKSPACE", "TQ_ERR_CUDA", "TQ_F32", "TQ_BF16", "TQ_LAYOUT_PLAIN", "TQ_LAYOUT_MIXED",
]
