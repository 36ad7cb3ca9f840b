"""Decode runs shared by the release library and the TQ_DEBUG build (tests/test_zw_debug_build.py):
the same seeded inputs through quantize, decode (four and eight heads per kv-head, ragged lengths,
many CTAs per unit), the fused decode step and the mixed layout.  Run as a script it writes the
outputs and the device error word of the library the environment selects to the file it is given."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
for p in (ROOT, os.path.dirname(os.path.abspath(__file__))):
    if p not in sys.path:
        sys.path.insert(0, p)

import decode_attention_11_b200 as tq  # noqa: E402
import workloads as W  # noqa: E402

from _parity import mixed_setup, params_for  # noqa: E402


def run_cases() -> dict:
    out = {}
    tq.reset_device_errors()
    # plain layout: small ragged case, and one long enough that every unit spans several CTAs
    for tag, name, over in (("b4", "llama3_8b_128k_b4", dict(T=531, B=2, Hkv=2, Hq=8)),
                            ("moe", "moe_1m", dict(T=900, B=1, Hkv=2, Hq=16)),
                            ("long", "llama3_8b_128k_b4", dict(T=20000, B=4, Hkv=8, Hq=32))):
        w = W.CONFIGS[name].scaled(**over)
        params = params_for(w)
        K, V = W.make_kv(w, "k").cuda(), W.make_kv(w, "v").cuda()
        cache = tq.Cache.allocate(w.B, w.Hkv, w.T + 3, w.k_bits, w.v_bits, w.qjl_m)
        tq.quantize(params, K, V, cache)
        q = W.make_queries(w).cuda()
        for L in (w.T, w.T - 37, 65, 1):
            out[f"{tag}_L{L}"] = tq.decode_attn(params, q, cache, L).cpu()
        # fused decode step on the rows after the quantized ones
        kn, vn = K[:, :, -1].contiguous(), V[:, :, -1].contiguous()
        for t in (w.T, w.T + 1):
            out[f"{tag}_step{t}"] = tq.decode_step(params, kn, vn, q, cache, t).cpu()
    # mixed layout
    w = W.CONFIGS["llama3_8b_128k_b4"].scaled(T=531, B=2, Hkv=2, Hq=8)
    oc, P, S = mixed_setup(w)
    params = tq.Params.create(P, S, 4, 4, outlier_channels=oc)
    K, V = W.make_kv(w, "k").cuda(), W.make_kv(w, "v").cuda()
    cache = tq.Cache.allocate(w.B, w.Hkv, w.T, 4, 4, w.qjl_m, layout=tq.TQ_LAYOUT_MIXED)
    tq.quantize(params, K, V, cache)
    q = W.make_queries(w).cuda()
    for L in (w.T, 100):
        out[f"mixed_L{L}"] = tq.decode_attn(params, q, cache, L).cpu()
    torch.cuda.synchronize()
    out["decode_errors"] = tq.decode_device_errors()
    out["quantize_errors"] = tq.quantize_device_errors()
    return out


if __name__ == "__main__":
    torch.save(run_cases(), sys.argv[1])
