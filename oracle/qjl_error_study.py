"""Attention-output error of the compressed cache against exact attention, with and without the
QJL term, for each workload recipe and both rotations (dense Haar, structured Hadamard).

The QJL term makes every score unbiased but adds variance, which the softmax can amplify
(ai-news.ru overview, paragraph on the third component); this measures that trade on the
synthetic workloads.  TEST INFRASTRUCTURE: it calls only the oracle and the input generator.

    python -m oracle.qjl_error_study [--T 2048]

Prints one Markdown table (float64 throughout; workloads cut to one batch, two kv-heads and T
tokens so that the oracle finishes in about a minute).
"""
import argparse
import dataclasses

import numpy as np

import workloads as W
from oracle import tq_oracle as O


def study(T: int):
    rows = []
    for name in W.CONFIG_ORDER:
        base = W.CONFIGS[name]
        hkv = min(2, base.Hkv)
        w0 = base.scaled(T=min(T, base.T), B=1, Hkv=hkv, Hq=base.group * hkv)
        for rotation in ("haar", "hadamard"):
            w = dataclasses.replace(w0, rotation=rotation)
            K = W.make_kv(w, "k").double().numpy()
            V = W.make_kv(w, "v").double().numpy()
            q = W.make_queries(w).double().numpy()
            Pi, S = W.rotation_for(w), W.qjl_for(w)
            exact = O.exact_attention(q, K, V)
            res = {}
            for label, sk in (("on", S), ("off", None)):
                cache = O.quantize_cache(K, V, Pi, w.k_bits, w.v_bits, sk)
                out = O.decode_attention(q, Pi, sk, cache, w.k_bits, w.v_bits, w.T)
                res[label] = (np.linalg.norm(out - exact) / np.linalg.norm(exact),
                              float(np.max(np.abs(out - exact))))
            rows.append((name, rotation, w.T, w.k_bits, w.v_bits, res["on"], res["off"]))
    return rows


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--T", type=int, default=2048)
    args = ap.parse_args()
    print("| workload | rotation | T | K/V bits | rel-L2, QJL on | rel-L2, QJL off | max-abs, QJL on | max-abs, QJL off |")
    print("|---|---|---:|---|---:|---:|---:|---:|")
    for name, rot, T, kb, vb, on, off in study(args.T):
        print(f"| {name} | {rot} | {T} | {kb}/{vb} | {on[0]:.4f} | {off[0]:.4f} | {on[1]:.4f} | {off[1]:.4f} |")


if __name__ == "__main__":
    main()
