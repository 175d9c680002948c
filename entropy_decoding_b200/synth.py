"""Seeded synthetic weights shaped like the LLM workloads of the DFloat11 page.

This module only draws numbers: it holds none of the compression method's
arithmetic, so both the CPU oracle (tests) and the product path (tests,
bench) can take their inputs from it.  Trained weights are not available, so
seeded draws with the workloads' shapes and value distributions stand in for
them ("70% Size, 100% Accuracy ... (DFloat11)", Abstract: Llama 3.x, Qwen 3,
Mistral 3 ... models).

Every tensor gets its own numpy ``Generator(PCG64)`` seeded by a child of
``SeedSequence(seed)``; children are spawned in a fixed tensor order.  FP32
draws are rounded to BF16 (or E4M3) round-to-nearest-even by torch on the CPU.
Weights are returned as their raw bit patterns: ``uint16`` for BF16,
``uint8`` for E4M3.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np
import torch

# Llama-3-8B-shaped transformer block, shapes written [in, out]: fan_in is the
# first dimension.
BLOCK_SHAPES = [
    ("q_proj", (4096, 4096)),
    ("k_proj", (4096, 1024)),
    ("v_proj", (4096, 1024)),
    ("o_proj", (4096, 4096)),
    ("gate_proj", (4096, 14336)),
    ("up_proj", (4096, 14336)),
    ("down_proj", (14336, 4096)),
]
N_BLOCKS = 32
VOCAB_SHAPE = (128256, 4096)


def _rng(ss: np.random.SeedSequence) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(ss))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """FP32 -> BF16 round-to-nearest-even (torch), returned as uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """FP32 -> FP8 E4M3 round-to-nearest-even (torch), returned as uint8 bits."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def normal_bf16(ss, n: int, std: float) -> np.ndarray:
    g = _rng(ss)
    x = g.standard_normal(n, dtype=np.float32)
    x *= np.float32(std)
    return to_bf16_bits(x)


def student_t_outliers_bf16(ss, n: int, scale: float = 0.02, df: float = 3.0,
                            outlier_frac: float = 1e-3) -> np.ndarray:
    """scale * t(df), with a Bernoulli(outlier_frac) subset replaced by N(0, 1)."""
    g = _rng(ss)
    x = (g.standard_t(df, n) * scale).astype(np.float32)
    mask = g.random(n) < outlier_frac
    x[mask] = g.standard_normal(int(mask.sum())).astype(np.float32)
    return to_bf16_bits(x)


def normal_e4m3(ss, n: int, std: float = 0.02) -> np.ndarray:
    """N(0, std) scaled per tensor so that max|x| maps to 448, then RNE."""
    g = _rng(ss)
    x = g.standard_normal(n, dtype=np.float32)
    x *= np.float32(std)  # in place: the same float32 products, no temporaries
    amax = max(float(x.max()), -float(x.min())) if n else 1.0
    x *= np.float32(448.0) / np.float32(amax)
    return to_e4m3_bits(x)


@dataclass
class Tensor:
    name: str
    shape: tuple
    bits: np.ndarray  # flat raw bit patterns


@dataclass
class Group:
    """Tensors sharing one code (one decode launch)."""
    name: str
    tensors: list


# ------------------------------------------------------------- workloads

def single_matrix(seed: int = 0) -> list[Group]:
    """1024x1024 BF16, iid N(0, 0.02)."""
    ss = np.random.SeedSequence(seed).spawn(1)[0]
    return [Group("m1024", [Tensor("w", (1024, 1024), normal_bf16(ss, 1024 * 1024, 0.02))])]


def heavy_tail_matrix(seed: int = 0) -> list[Group]:
    """4096x4096 BF16, 0.02 * Student-t(3) plus 0.1% N(0, 1) outliers."""
    ss = np.random.SeedSequence(seed).spawn(1)[0]
    n = 4096 * 4096
    return [Group("t4096", [Tensor("w", (4096, 4096), student_t_outliers_bf16(ss, n))])]


def _block_tensors(children, workers: int | None):
    def one(i):
        name, shape = BLOCK_SHAPES[i]
        n = shape[0] * shape[1]
        return Tensor(name, shape, normal_bf16(children[i], n, 1.0 / math.sqrt(shape[0])))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        return list(ex.map(one, range(len(BLOCK_SHAPES))))


def transformer_block(seed: int = 0, workers: int | None = None) -> list[Group]:
    """One Llama-3-8B-shaped block, each matrix N(0, 1/sqrt(fan_in))."""
    children = np.random.SeedSequence(seed).spawn(len(BLOCK_SHAPES))
    return [Group("block0", _block_tensors(children, workers))]


def whole_model_specs():
    """(group name, [(tensor name, shape, kind)]) for the whole model, in
    decode order: embedding, 32 blocks, LM head."""
    specs = [("embed", [("embed_tokens", VOCAB_SHAPE, "normal002")])]
    for b in range(N_BLOCKS):
        specs.append((f"block{b}", [(n, s, "fanin") for n, s in BLOCK_SHAPES]))
    specs.append(("lm_head", [("lm_head", VOCAB_SHAPE, "normal002")]))
    return specs


def whole_model_group(seed: int, gi: int) -> Group:
    """Group gi of the whole model.  Seeds: SeedSequence(seed).spawn(34)[gi],
    then one child per tensor of the group."""
    specs = whole_model_specs()
    gname, tspecs = specs[gi]
    gss = np.random.SeedSequence(seed).spawn(len(specs))[gi]
    children = gss.spawn(len(tspecs))

    def one(i):
        name, shape, kind = tspecs[i]
        n = shape[0] * shape[1]
        std = 0.02 if kind == "normal002" else 1.0 / math.sqrt(shape[0])
        return Tensor(name, shape, normal_bf16(children[i], n, std))

    with ThreadPoolExecutor() as ex:
        return Group(gname, list(ex.map(one, range(len(tspecs)))))


def e4m3_matrix(seed: int = 0) -> list[Group]:
    """8192x28672 FP8 E4M3, N(0, 0.02) scaled to the E4M3 range."""
    ss = np.random.SeedSequence(seed).spawn(1)[0]
    n = 8192 * 28672
    return [Group("e4m3", [Tensor("w", (8192, 28672), normal_e4m3(ss, n))])]


# ------------------------------------------------------------- adversarial inputs

def all_bf16_patterns() -> np.ndarray:
    """Every 16-bit pattern once (+-0, subnormals, +-inf, NaN payloads)."""
    return np.arange(65536, dtype=np.uint32).astype(np.uint16)


def all_e4m3_patterns() -> np.ndarray:
    return np.arange(256, dtype=np.uint16).astype(np.uint8)


def constant_bf16(n: int, value: float = 0.0) -> np.ndarray:
    return to_bf16_bits(np.full(n, value, np.float32))


def powers_of_two_bf16(counts, first_exponent: int = -30, seed: int = 0) -> np.ndarray:
    """A shuffled tensor holding counts[k] values of magnitude in
    [2^(first_exponent+k), 2^(first_exponent+k+1)), with random sign and
    random 7-bit fraction.  Every value is exactly representable in BF16, so
    the tensor's binary exponents follow the given histogram."""
    g = _rng(np.random.SeedSequence(seed))
    parts = []
    for k, c in enumerate(counts):
        c = int(c)
        frac = 1.0 + g.integers(0, 128, c).astype(np.float32) / np.float32(128.0)
        sign = np.where(g.random(c) < 0.5, -1.0, 1.0).astype(np.float32)
        parts.append(np.ldexp(frac, first_exponent + k).astype(np.float32) * sign)
    x = np.concatenate(parts) if parts else np.zeros(0, np.float32)
    g.shuffle(x)
    return to_bf16_bits(x)


def fibonacci_counts(k: int = 34) -> list[int]:
    f = [1, 1]
    while len(f) < k:
        f.append(f[-1] + f[-2])
    return f[:k]


def random_bits(n: int, dtype: str, seed: int = 0) -> np.ndarray:
    """Uniformly random bit patterns (a flat exponent histogram)."""
    g = _rng(np.random.SeedSequence(seed))
    if dtype == "bf16":
        return g.integers(0, 65536, n, dtype=np.uint32).astype(np.uint16)
    return g.integers(0, 256, n, dtype=np.uint16).astype(np.uint8)
