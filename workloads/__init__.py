"""Seeded synthetic inputs for the low-bit linear layer.

This module draws random numbers and nothing else: no packing, no
dequantisation, no matrix product.  Tests, the smoke check and the benchmark
feed the same arrays to the CPU oracle and to the CUDA library.

Distributions follow the workloads the pages describe for Bonsai Image 4B
(a 25-block MMDiT with hidden size 3072, 1024 image tokens at 512x512 and
4096 at 1024x1024 plus text tokens):
  - activations A ~ N(0, 1), rounded to FP16;
  - ternary codes with P(0) = 0.4, P(+1) = P(-1) = 0.3;
  - binary codes +1 / -1 with probability 1/2 each;
  - scales ~ U[0.005, 0.05], rounded to FP16, one per 128 weights along K.
Every stream comes from numpy's PCG64 seeded through a SeedSequence; the
activations, codes and scales use three spawned child streams so that each
is independent of the others' sizes.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

GROUP = 128


@dataclass(frozen=True)
class Problem:
    name: str
    mode: str  # "binary" | "ternary" (INT2) | "ternary_b3" (base-3 storage of the same codes)
    M: int
    N: int
    K: int
    seed: int


# The configurations the parity tests and the benchmark use.
TERNARY_TINY = Problem("ternary tiny", "ternary", 64, 256, 256, 1001)
BINARY_512_LINEAR = Problem("binary 512^2-image linear", "binary", 1024, 3072, 3072, 1002)
TERNARY_MLP_UP_4608 = Problem("ternary 1024^2+text MLP-up", "ternary", 4608, 9216, 3072, 1003)
TERNARY_MLP_DOWN_4608 = Problem("ternary MLP-down M=4608", "ternary", 4608, 3072, 9216, 1004)
TERNARY_QKV_4608 = Problem("ternary fused QKV M=4608", "ternary", 4608, 9216, 3072, 1005)
TERNARY_MLP_DOWN_16 = Problem("ternary MLP-down M=16", "ternary", 16, 3072, 9216, 1014)
TERNARY_QKV_16 = Problem("ternary fused QKV M=16", "ternary", 16, 9216, 3072, 1015)

CONFIGS = [
    TERNARY_TINY,
    BINARY_512_LINEAR,
    TERNARY_MLP_UP_4608,
    TERNARY_MLP_DOWN_4608,
    TERNARY_QKV_4608,
    TERNARY_MLP_DOWN_16,
    TERNARY_QKV_16,
]


def mmdit_stack_layers(hidden: int = 3072, split_qkv: bool = False):
    """(name, N, K) of the low-bit linears in one denoise step of a 25-block
    MMDiT: 5 double-stream blocks (two streams each with QKV, attention-out,
    MLP-up, MLP-down) and 20 single-stream blocks (fused QKV+MLP-up, fused
    out).  With Q|K|V stacked, 80 launches cover the 100 linears; with
    split_qkv the double-stream Q, K and V are separate launches (100)."""
    h = hidden
    layers = []
    for b in range(5):
        for stream in ("img", "txt"):
            if split_qkv:
                layers += [(f"double{b}.{stream}.{x}", h, h) for x in ("q", "k", "v")]
            else:
                layers.append((f"double{b}.{stream}.qkv", 3 * h, h))
            layers.append((f"double{b}.{stream}.out", h, h))
            layers.append((f"double{b}.{stream}.mlp_up", 3 * h, h))
            layers.append((f"double{b}.{stream}.mlp_down", h, 3 * h))
    for b in range(20):
        layers.append((f"single{b}.qkv_mlp_up", 6 * h, h))
        layers.append((f"single{b}.out", h, 4 * h))
    return layers


def mmdit_stream_layers(img_tokens: int, txt_tokens: int, hidden: int = 3072):
    """(name, M, N, K) of the low-bit linears in one denoise step with the
    real per-stream token counts: the double-stream blocks run their image
    and text streams as separate linears (separate weights) on img_tokens and
    txt_tokens rows, the single-stream blocks on the joint sequence.  1024^2
    images give 4096 image tokens, 512^2 give 1024; the text stream is 512."""
    joint = img_tokens + txt_tokens
    out = []
    for name, n, k in mmdit_stack_layers(hidden):
        if name.startswith("double"):
            out.append((name, img_tokens if ".img." in name else txt_tokens, n, k))
        else:
            out.append((name, joint, n, k))
    return out


def _streams(seed: int):
    ss = np.random.SeedSequence(seed)
    return [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(3)]


def activations(rng: np.random.Generator, M: int, K: int) -> np.ndarray:
    """fp16 bit patterns (uint16) of N(0,1) draws, [M,K]."""
    return rng.standard_normal((M, K), dtype=np.float64).astype(np.float16).view(np.uint16)


def codes(rng: np.random.Generator, N: int, K: int, mode: str) -> np.ndarray:
    """int8 weight codes [N,K]."""
    u = rng.random((N, K), dtype=np.float64)
    if mode == "binary":
        return np.where(u < 0.5, 1, -1).astype(np.int8)
    if mode in ("ternary", "ternary_b3"):  # one code alphabet, two storage formats
        return np.where(u < 0.3, -1, np.where(u < 0.7, 0, 1)).astype(np.int8)
    raise ValueError(mode)


def scales(rng: np.random.Generator, N: int, K: int) -> np.ndarray:
    """fp16 bit patterns (uint16) of U[0.005, 0.05] draws, [N, K/128]."""
    return rng.uniform(0.005, 0.05, (N, K // GROUP)).astype(np.float16).view(np.uint16)


def make_hqq4(M: int, N: int, K: int, seed: int):
    """Inputs for the 4-bit group-affine weights: A (uint16 fp16 bits [M,K]),
    q (uint8 [N,K], uniform on 0..15), scales ~ U[0.005, 0.05] and zeros ~
    U[0, 15] (fp16 bits [N, K/64]), from the same spawned-stream scheme."""
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    ra, rc, rs = _streams(seed)
    return {
        "M": M, "N": N, "K": K,
        "A": activations(ra, M, K),
        "q": rc.integers(0, 16, (N, K), dtype=np.uint8),
        "scales": rs.uniform(0.005, 0.05, (N, K // 64)).astype(np.float16).view(np.uint16),
        "zeros": rs.uniform(0.0, 15.0, (N, K // 64)).astype(np.float16).view(np.uint16),
    }


def make(problem: Problem | None = None, *, mode=None, M=None, N=None, K=None, seed=None):
    """-> dict with A (uint16 fp16 bits [M,K]), codes (int8 [N,K]),
    scales (uint16 fp16 bits [N,K/128]) and the problem's sizes."""
    if problem is not None:
        mode, M, N, K, seed = problem.mode, problem.M, problem.N, problem.K, problem.seed
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    ra, rc, rs = _streams(seed)
    return {
        "mode": mode,
        "M": M,
        "N": N,
        "K": K,
        "A": activations(ra, M, K),
        "codes": codes(rc, N, K, mode),
        "scales": scales(rs, N, K),
    }
