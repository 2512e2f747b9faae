"""Seeded synthetic inputs for the weight-quantised GEMM workloads.

This module only draws random numbers and casts them to the storage types
(fp32 weights, bf16 activations and biases). It holds none of the method's
arithmetic: no packing, no dequantisation, no matmul. Both the oracle and the
CUDA path take their inputs from here.

Shapes follow FLUX.1's double-stream transformer linears: hidden width 3072,
MLP width 12288, 4096 image tokens for a 1024x1024 picture (mflux-rs landing
page, "Patch Packing & Memory Calculator": 128x128 latents -> 64x64 patches ->
4,096 image tokens) plus 512 text tokens for the MLP pair. Trained FLUX
weights are not available, so every tensor is drawn from a fixed distribution
with a fixed seed; the distributions are stated per linear below.

bf16 casts use torch's CPU conversion (round to nearest even), a library
routine; fp16 casts of the ternary scales use numpy's.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Linear:
    """One quantised linear layer: out[M,N] = X[M,K] . dequant(W)[N,K]^T (+ bias)."""
    name: str
    M: int
    N: int
    K: int
    bits: int            # 1 = 1-bit, 2 = ternary, 4 or 8 = group-wise affine
    group: int           # 64 for affine, 128 for ternary and 1-bit
    bias: bool           # bf16 bias [N] ~ N(0, 0.01)
    x_dist: str          # "normal" = N(0,1); "gelu" = tanh-GELU of N(0,1)
    w_dist: str          # "normal" = N(0, 0.02) fp32; "ternary" = s16 * t

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


@dataclasses.dataclass(frozen=True)
class Workload:
    cid: int
    name: str
    linears: tuple


def _aff(name, M, N, K, bits, bias=False, x="normal"):
    return Linear(name, M, N, K, bits, 64, bias, x, "normal")


def _tern(name, M, N=12288, K=3072):
    return Linear(name, M, N, K, 2, 128, False, "normal", "ternary")


def _bin(name, M, N=12288, K=3072):
    return Linear(name, M, N, K, 1, 128, False, "normal", "binary")


WORKLOADS = (
    Workload(0, "tiny 4-bit [64,512]x[512,512]",
             (_aff("tiny", 64, 512, 512, 4),)),
    Workload(1, "FLUX double-stream image QKV [4096,3072]x[9216,3072] 4-bit + bias",
             (_aff("qkv", 4096, 9216, 3072, 4, bias=True),)),
    Workload(2, "FLUX MLP pair, 4608 tokens: up 4-bit [4608,3072]x[12288,3072], "
                "down 8-bit [4608,12288]x[3072,12288]",
             (_aff("mlp_up", 4608, 12288, 3072, 4),
              _aff("mlp_down", 4608, 3072, 12288, 8, x="gelu"))),
    Workload(3, "ternary small-M sweep M in {1,4,16}, [M,3072]x[12288,3072]",
             (_tern("tern_m1", 1), _tern("tern_m4", 4), _tern("tern_m16", 16))),
    Workload(4, "mixed FLUX double-stream block linears, M=4608: residual-writing "
                "8-bit, the rest 4-bit",
             (_aff("modulation", 4608, 18432, 3072, 8),
              _aff("qkv", 4608, 9216, 3072, 4),
              _aff("out_proj", 4608, 3072, 3072, 8),
              _aff("mlp_up", 4608, 12288, 3072, 4),
              _aff("mlp_down", 4608, 3072, 12288, 8, x="gelu"))),
    Workload(5, "sub-byte formats at DiT shapes: ternary prefill M=4096 and 1-bit (Q1_0_g128) decode M=1 and "
                "prefill M=4096, [M,3072]x[12288,3072]",
             (_tern("tern_prefill", 4096), _bin("bin_m1", 1), _bin("bin_prefill", 4096))),
)


def workload(cid: int) -> Workload:
    return WORKLOADS[cid]


# tensor ids inside the seed sequence
_T_X, _T_W, _T_BIAS, _T_SCALE, _T_TERN = 1, 2, 3, 4, 5


def _rng(cid: int, lin_idx: int, tensor: int, extra: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([0, cid, lin_idx, tensor, extra]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 storage bits (uint16) through torch's CPU conversion."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 storage bits -> fp32 values (exact widening)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """tanh-approximate GELU in fp64; only shapes the input distribution."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def make_x(cid: int, lin_idx: int, M: int, K: int, dist: str, extra: int = 0) -> np.ndarray:
    """Activations as bf16 bits [M, K]."""
    x = _rng(cid, lin_idx, _T_X, extra).standard_normal((M, K))
    if dist == "gelu":
        x = gelu_tanh(x)
    elif dist != "normal":
        raise ValueError(dist)
    return f32_to_bf16_bits(x.astype(np.float32))


def make_w(cid: int, lin_idx: int, N: int, K: int, dist: str, group: int = 128,
           extra: int = 0) -> np.ndarray:
    """Weights as fp32 [N, K].

    "normal": N(0, 0.02).  "ternary": W = fp32(s16) * t with t uniform on
    {-1, 0, +1} (P(0) = 1/3) and one fp16 scale s16 ~ U(0.01, 0.05) per group
    of `group` consecutive k, so the weights are exactly representable by the
    ternary format.  "binary": the same with signs uniform on {-1, +1}, exactly
    representable by the 1-bit format.
    """
    if dist == "normal":
        return (_rng(cid, lin_idx, _T_W, extra).standard_normal((N, K)) * 0.02).astype(np.float32)
    if dist == "ternary":
        t = _rng(cid, lin_idx, _T_TERN, extra).integers(-1, 2, size=(N, K)).astype(np.float32)
        s = _rng(cid, lin_idx, _T_SCALE, extra).uniform(0.01, 0.05, size=(N, K // group))
        s16 = s.astype(np.float16).astype(np.float32)
        return (t * np.repeat(s16, group, axis=1)).astype(np.float32)
    if dist == "binary":
        c = 2.0 * _rng(cid, lin_idx, _T_TERN, extra).integers(0, 2, size=(N, K)).astype(np.float32) - 1.0
        s = _rng(cid, lin_idx, _T_SCALE, extra).uniform(0.01, 0.05, size=(N, K // group))
        s16 = s.astype(np.float16).astype(np.float32)
        return (c * np.repeat(s16, group, axis=1)).astype(np.float32)
    raise ValueError(dist)


def make_bias(cid: int, lin_idx: int, N: int, extra: int = 0) -> np.ndarray:
    """bf16 bits [N] ~ N(0, 0.01)."""
    b = _rng(cid, lin_idx, _T_BIAS, extra).standard_normal(N) * 0.01
    return f32_to_bf16_bits(b.astype(np.float32))


def make_inputs(lin: Linear, cid: int, lin_idx: int, M: Optional[int] = None, extra: int = 0):
    """(X bf16 bits [M,K], W fp32 [N,K], bias bf16 bits [N] or None) for one linear."""
    M = lin.M if M is None else M
    X = make_x(cid, lin_idx, M, lin.K, lin.x_dist, extra)
    W = make_w(cid, lin_idx, lin.N, lin.K, lin.w_dist, lin.group, extra)
    bias = make_bias(cid, lin_idx, lin.N, extra) if lin.bias else None
    return X, W, bias


def random_case(seed: int, M: int, N: int, K: int, bits: int, with_bias: bool,
                x_scale: float = 1.0, w_scale: float = 0.02):
    """A seeded off-config case (ragged sizes, edge tests)."""
    g = np.random.default_rng(np.random.SeedSequence([1, seed, M, N, K, bits]))
    X = f32_to_bf16_bits((g.standard_normal((M, K)) * x_scale).astype(np.float32))
    if bits == 1:
        c = 2.0 * g.integers(0, 2, size=(N, K)).astype(np.float32) - 1.0
        s16 = g.uniform(0.01, 0.05, size=(N, K // 128)).astype(np.float16).astype(np.float32)
        W = (c * np.repeat(s16, 128, axis=1)).astype(np.float32)
    elif bits == 2:
        t = g.integers(-1, 2, size=(N, K)).astype(np.float32)
        s16 = g.uniform(0.01, 0.05, size=(N, K // 128)).astype(np.float16).astype(np.float32)
        W = (t * np.repeat(s16, 128, axis=1)).astype(np.float32)
    else:
        W = (g.standard_normal((N, K)) * w_scale).astype(np.float32)
    bias = f32_to_bf16_bits((g.standard_normal(N) * 0.01).astype(np.float32)) if with_bias else None
    return X, W, bias
