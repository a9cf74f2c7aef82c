"""Synthetic parameter sets of the workloads: shapes only (no weights, no data).

Llama-2-7B / 13B parameter lists in module order (token embedding; per layer q,
k, v, o, gate, up, down projections and the two RMSNorm weights; final norm;
lm_head), the 10,000-tensor ragged set, and the 1-tensor tiny set.
"""
from __future__ import annotations

import numpy as np


def llama_shapes(hidden, inter, layers, vocab=32000):
    out = [("embed_tokens", vocab * hidden)]
    for i in range(layers):
        p = "layers.%d." % i
        out += [(p + "q_proj", hidden * hidden), (p + "k_proj", hidden * hidden),
                (p + "v_proj", hidden * hidden), (p + "o_proj", hidden * hidden),
                (p + "gate_proj", inter * hidden), (p + "up_proj", inter * hidden),
                (p + "down_proj", hidden * inter), (p + "input_layernorm", hidden),
                (p + "post_attention_layernorm", hidden)]
    out += [("norm", hidden), ("lm_head", vocab * hidden)]
    return out


def llama2_7b():
    return llama_shapes(4096, 11008, 32)


def llama2_13b():
    return llama_shapes(5120, 13824, 40)


def tiny():
    return [("flat", 1 << 20)]


def ragged(num=10000, lo=64, hi=1 << 20, seed=0):
    """Sizes log-uniform in [lo, hi] (integers, generally not multiples of 128)."""
    rng = np.random.default_rng(seed)
    sizes = np.exp(rng.uniform(np.log(lo), np.log(hi), num)).astype(np.int64)
    return [("t%d" % i, int(s)) for i, s in enumerate(sizes)]


def flat(n):
    return lambda: [("flat", n)]


CONFIGS = {
    "flat-256m": dict(shapes=flat(1 << 28), fmt_m=0, fmt_v=1, steps=3,
                      workload="One flat tensor of 268,435,456 params, E4M3 m + E5M2 v "
                               "(profiling case: 2.7 GB, larger than L2)"),
    "tiny": dict(shapes=tiny, fmt_m=0, fmt_v=0, steps=10,
                 workload="Tiny: one flat tensor of 1,048,576, E4M3 m + E4M3 v"),
    "llama2-7b": dict(shapes=llama2_7b, fmt_m=0, fmt_v=1, steps=3,
                      workload="Llama-2-7B-shaped parameter list (291 tensors, 6,738,415,616 "
                               "params), E4M3 m + E5M2 v"),
    "llama2-13b": dict(shapes=llama2_13b, fmt_m=0, fmt_v=0, steps=1,
                       workload="Llama-2-13B-shaped parameter list (363 tensors, 13,015,864,320 "
                                "params), E4M3 m + E4M3 v"),
    "ragged": dict(shapes=ragged, fmt_m=0, fmt_v=1, steps=3,
                   workload="Ragged: 10,000 tensors, sizes log-uniform in [64, 1,048,576], "
                            "E4M3 m + E5M2 v"),
}

# AdamW hyperparameters of the workloads
HYPER = dict(lr=1e-4, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)
