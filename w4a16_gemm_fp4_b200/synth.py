"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle
checks.

This module draws random numbers and nothing else: it holds none of the
quantization or GEMM arithmetic.  Every workload is a numpy PCG64 stream
(``numpy.random.default_rng(seed)``) drawn in the order written below, so
the same seed gives the same tensors on any machine.  Activations are drawn
in fp32 and rounded to bf16 by torch's round-to-nearest-even cast; they are
returned as uint16 bit patterns.

Workloads (shapes of LLaMA-7B / LLaMA-13B linear layers, the models the
pages measure on; no trained weights exist here, so seeded draws stand in):

* ``tiny``            W 256x512 ~ N(0, 0.02^2); x 1x512 ~ N(0, 1); seed 0.
* ``llama7b_decode``  W 4096x4096, 11008x4096, 4096x11008 ~ N(0, 0.02^2)
                      times a per-row lognormal(0, 0.3) factor; X with
                      M in {1, 8, 16, 64} rows ~ N(0, 1); seed 1.
* ``llama7b_prefill`` W 4096x4096 and 11008x4096 as above; X 2048x4096
                      ~ N(0, 1) with 41 (1 %) input channels, chosen once by
                      ``rng.choice(K, 41, replace=False)``, scaled by 50; seed 2.
* ``llama13b_search`` W 5120x5120 and 13824x5120 ~ 0.015 * Student-t(5);
                      X 512x5120 ~ N(0, 1); seed 3.
* ``llama13b_stack``  40 layers x {q,k,v,o 5120x5120, gate,up 13824x5120,
                      down 5120x13824} ~ N(0, 0.02^2), drawn on the GPU with
                      ``torch.Generator('cuda').manual_seed(4)`` because 50 GB
                      of fp32 host draws is impractical.
"""
from __future__ import annotations

import numpy as np
import torch

LLAMA7B_DECODE_SHAPES = ((4096, 4096), (11008, 4096), (4096, 11008))
LLAMA7B_DECODE_MS = (1, 8, 16, 64)
LLAMA7B_PREFILL_SHAPES = ((4096, 4096), (11008, 4096))
LLAMA13B_SEARCH_SHAPES = ((5120, 5120), (13824, 5120))
LLAMA13B_LAYER_SHAPES = (("q", 5120, 5120), ("k", 5120, 5120), ("v", 5120, 5120), ("o", 5120, 5120),
                         ("gate", 13824, 5120), ("up", 13824, 5120), ("down", 5120, 13824))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), torch RNE cast."""
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_weights(rng, N, K, std=0.02):
    return rng.standard_normal((N, K), dtype=np.float32) * np.float32(std)


def lognormal_row_weights(rng, N, K):
    W = normal_weights(rng, N, K)
    rowf = rng.lognormal(0.0, 0.3, N).astype(np.float32)
    return W * rowf[:, None]


def student_t_weights(rng, N, K, nu=5, scale=0.015):
    return (rng.standard_t(nu, size=(N, K)) * scale).astype(np.float32)


def activations(rng, M, K):
    return to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32))


def tiny(seed=0):
    rng = np.random.default_rng(seed)
    W = normal_weights(rng, 256, 512)
    X = activations(rng, 1, 512)
    return {"W": W, "X": X}


def llama7b_decode(seed=1, shapes=LLAMA7B_DECODE_SHAPES, ms=LLAMA7B_DECODE_MS):
    """Returns list of dicts {W, X: {M: bits}} in shape order."""
    rng = np.random.default_rng(seed)
    out = []
    for (N, K) in shapes:
        W = lognormal_row_weights(rng, N, K)
        X = {M: activations(rng, M, K) for M in ms}
        out.append({"W": W, "X": X})
    return out


def outlier_activations(rng, M, K, frac=0.01, factor=50.0):
    n_out = int(round(K * frac))
    idx = rng.choice(K, n_out, replace=False)
    X = rng.standard_normal((M, K), dtype=np.float32)
    X[:, idx] *= np.float32(factor)
    return to_bf16_bits(X), np.sort(idx)


def llama7b_prefill(seed=2, M=2048, shapes=LLAMA7B_PREFILL_SHAPES):
    rng = np.random.default_rng(seed)
    K = shapes[0][1]
    X, idx = outlier_activations(rng, M, K)
    Ws = [lognormal_row_weights(rng, N, Kw) for (N, Kw) in shapes]
    return {"X": X, "outlier_channels": idx, "W": Ws}


def llama13b_search(seed=3, M=512, shapes=LLAMA13B_SEARCH_SHAPES):
    rng = np.random.default_rng(seed)
    Ws = [student_t_weights(rng, N, K) for (N, K) in shapes]
    X = activations(rng, M, shapes[0][1])
    return {"W": Ws, "X": X}


def random_case(seed, N, K, M, dist="normal"):
    """Small seeded case for parity tests: W [N][K] fp32, X [M][K] bf16 bits."""
    rng = np.random.default_rng(seed)
    if dist == "t":
        W = student_t_weights(rng, N, K)
    elif dist == "lognormal_rows":
        W = lognormal_row_weights(rng, N, K)
    else:
        W = normal_weights(rng, N, K)
    X = activations(rng, M, K)
    return W, X


def stack_layer_weights(layer: int, device="cuda", seed=4):
    """Weights of one layer of the 13B-shaped stack, drawn on the GPU.

    Each layer reseeds with seed * 1000 + layer so that any layer can be
    regenerated alone (the parity test samples layers)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + layer)
    out = []
    for (name, N, K) in LLAMA13B_LAYER_SHAPES:
        w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * 0.02
        out.append((name, w))
    return out
