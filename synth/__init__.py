"""Seeded synthetic inputs for the 4-bit codebook linear layer.

This module serves both the CUDA path (tests, bench, smoke) and the oracle.
It holds none of the method's arithmetic.  It draws random numbers, converts
samples to the storage formats the layer takes (binary16, bfloat16 bit
patterns), and lists the layer shapes of the workloads.  Quantization,
dequantization and the matmul live elsewhere: in the oracle and in the CUDA
library, separately.

Workloads (Llama layer shapes, K -> N, tokens M):
  tiny              one layer 256 -> 128, M = 1; codes uniform in 0..15 (so
                    code bytes are uniform in 0..255), scales U[0.005, 0.05]
                    rounded to binary16, x ~ N(0,1) in bfloat16
  llama2_7b_layer   qkv 4096->12288, o 4096->4096, gate_up 4096->22016,
                    down 11008->4096; M = 1; W ~ N(0, 0.02) in fp32 from seed,
                    quantized by the layer's own pack step
  llama31_8b_step   32 x (qkv 4096->6144, o 4096->4096, gate_up 4096->28672,
                    down 14336->4096) + lm_head 4096->128256; M = 1
  small_m_verify    the Llama-3.1-8B linears + lm_head at M in {2, 4, 8, 16}
  llama2_70b_prefill qkv 8192->10240, o 8192->8192, gate_up 8192->57344,
                    down 28672->8192; W ~ N(0, 0.01); M in {32, 128, 256, 512}

Seeds: seed = 1000 * workload_index + 10 * layer + linear_index
(qkv 0, o 1, gate_up 2, down 3, lm_head 4); x draws use seed + 500000.
The generator is numpy's PCG64; normal samples come out in float32.
"""
from __future__ import annotations

import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
CODEBOOK_FILE = os.path.join(os.path.dirname(_HERE), "tests", "golden", "nf4_codebook.txt")

LINEAR_INDEX = {"qkv": 0, "o": 1, "gate_up": 2, "down": 3, "lm_head": 4}


@dataclass(frozen=True)
class Linear:
    name: str
    K: int
    N: int


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    linears: tuple
    Ms: tuple
    w_std: float
    layers: int = 1


LLAMA2_7B = (Linear("qkv", 4096, 12288), Linear("o", 4096, 4096),
             Linear("gate_up", 4096, 22016), Linear("down", 11008, 4096))
LLAMA31_8B = (Linear("qkv", 4096, 6144), Linear("o", 4096, 4096),
              Linear("gate_up", 4096, 28672), Linear("down", 14336, 4096))
LLAMA31_8B_HEAD = Linear("lm_head", 4096, 128256)
LLAMA2_70B = (Linear("qkv", 8192, 10240), Linear("o", 8192, 8192),
              Linear("gate_up", 8192, 57344), Linear("down", 28672, 8192))

WORKLOADS = {
    "tiny": Workload(0, "tiny", (Linear("tiny", 256, 128),), (1,), 0.0),
    "llama2_7b_layer": Workload(1, "llama2_7b_layer", LLAMA2_7B, (1,), 0.02),
    "llama31_8b_step": Workload(2, "llama31_8b_step", LLAMA31_8B + (LLAMA31_8B_HEAD,), (1,), 0.02,
                                layers=32),
    "small_m_verify": Workload(3, "small_m_verify", LLAMA31_8B + (LLAMA31_8B_HEAD,), (2, 4, 8, 16),
                               0.02),
    "llama2_70b_prefill": Workload(4, "llama2_70b_prefill", LLAMA2_70B, (32, 128, 256, 512), 0.01),
}


def seed_for(workload_index: int, layer: int, linear_name: str) -> int:
    return 1000 * workload_index + 10 * layer + LINEAR_INDEX.get(linear_name, 0)


def x_seed(seed: int) -> int:
    return seed + 500000


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round float32 samples to bfloat16 (nearest, ties to even); finite inputs."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def f32_to_f16_bits(f: np.ndarray) -> np.ndarray:
    """Round float32 samples to binary16 with numpy's own conversion."""
    return np.ascontiguousarray(f, dtype=np.float32).astype(np.float16).view(np.uint16)


def weights(seed: int, N: int, K: int, std: float) -> np.ndarray:
    """W [N, K] float32 ~ N(0, std^2)."""
    w = _rng(seed).standard_normal((N, K), dtype=np.float32)
    w *= np.float32(std)
    return w


def activations(seed: int, M: int, K: int) -> np.ndarray:
    """x [M, K] as bfloat16 bit patterns, x ~ N(0, 1)."""
    return f32_to_bf16_bits(_rng(seed).standard_normal((M, K), dtype=np.float32))


def tiny_codes_scales(seed: int, N: int, K: int):
    """Uniform 4-bit codes (two per byte) and binary16 scales U[0.005, 0.05]."""
    r = _rng(seed)
    codes = r.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = f32_to_f16_bits(r.uniform(0.005, 0.05, size=(N, K // 64)).astype(np.float32))
    return codes, scales


def tiny_codes2_scales(seed: int, N: int, K: int):
    """Uniform 2-bit codes (four per byte, every byte value equally likely)
    and binary16 scales U[0.005, 0.05], for the two-bit variant."""
    r = _rng(seed)
    codes = r.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    scales = f32_to_f16_bits(r.uniform(0.005, 0.05, size=(N, K // 64)).astype(np.float32))
    return codes, scales


def codebook2() -> np.ndarray:
    """A synthetic 4-entry codebook for the two-bit variant, as binary16 bit
    patterns: -1, -1/3, 1/3, 1 (each rounded to binary16)."""
    return np.array([-1.0, -1.0 / 3.0, 1.0 / 3.0, 1.0], dtype=np.float16).view(np.uint16)


def codebook() -> np.ndarray:
    """The NF4 codebook as 16 binary16 bit patterns, read from the committed fixture."""
    vals = []
    with open(CODEBOOK_FILE) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                vals.append(int(line.split()[0], 16))
    if len(vals) != 16:
        raise RuntimeError(f"{CODEBOOK_FILE}: expected 16 entries, found {len(vals)}")
    return np.array(vals, dtype=np.uint16)


def weights_device(seed: int, N: int, K: int, std: float, device):
    """W [N, K] float32 ~ N(0, std^2) drawn on a CUDA device with torch's seeded
    generator (Philox); used where host generation of hundreds of millions of
    samples would dominate the run time.  Same distribution as ``weights``,
    different stream."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
    return w.mul_(std)


def activations_device(seed: int, M: int, K: int, device):
    """x [M, K] bfloat16 ~ N(0, 1) drawn on a CUDA device (rounded to nearest-even)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn((M, K), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def integer_codebook() -> np.ndarray:
    """Codebook {-8, ..., 7} (exact in binary16), used for exact-arithmetic checks."""
    return f32_to_f16_bits(np.arange(-8, 8, dtype=np.float32))
