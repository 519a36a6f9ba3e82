"""Seeded synthetic inputs for the Strata MoE layer.

This module is the one piece shared by the CPU oracle's tests and the CUDA
path's tests and bench: it only draws random numbers and lays them out in the
canonical packed format.  It holds none of the layer's arithmetic (no
dequantisation, no routing, no FFN).

Workload recipe (the layer shapes follow the Qwen3.8-Flash-Next model as the
pages describe it: "Strata Runs 125B Qwen3.8-Flash-Next on a 12GB Gaming GPU at
Up to 94 Tokens/s", section "What it is": 48 layers x 512 experts, 10 routed +
1 shared per token; "Strata ... gaming PC" spec table: hidden dimension 2,560):

* hidden states: N(0, 1) rounded to bf16 (round to nearest even);
* router weight W_r [E, H]: N(0, 1/H) in fp32 (variance 1/H);
* router bias b [E] (optional): 0.5 * ln(Zipf(s=1.1) pmf at the expert's
  popularity rank), ranks given by a seeded permutation of 1..E;
* expert codes: uniform random bits, i.e. every code q uniform in 0..2^bits-1;
* block scales d [rows, cols/32]: exp(N(ln 0.02, 0.3)) rounded to fp16.

Canonical packed format (the C-ABI input format, see include/strata_moe.h):

* codes  uint8  [E][3][rows][cols/32][4*bits]  mats: 0 gate [I,H], 1 up [I,H],
  2 down [H,I]; every mat holds I*H weights so the per-mat stride is uniform;
* scales uint16 [E][3][rows][cols/32]  (fp16 bit patterns).

Random streams: numpy PCG64, keyed by SeedSequence([seed, layer, tensor, chunk])
so that each tensor of each layer is an independent stream and large tensors
can be drawn in parallel chunks without changing the result.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

# tensor ids of the independent streams
T_HIDDEN, T_ROUTER_W, T_ROUTER_B, T_CODES, T_SCALES, T_SH_CODES, T_SH_SCALES = range(1, 8)

_CHUNK = 1 << 22


@dataclass(frozen=True)
class LayerShape:
    hidden: int
    n_experts: int
    top_k: int
    inter: int
    bits: int = 2
    router_bias: bool = False

    @property
    def mat_weights(self) -> int:
        return self.hidden * self.inter

    @property
    def mat_code_bytes(self) -> int:
        return self.mat_weights * self.bits // 8

    @property
    def mat_scales(self) -> int:
        return self.mat_weights // 32

    @property
    def expert_bytes(self) -> int:
        return 3 * (self.mat_code_bytes + 2 * self.mat_scales)


# The five workloads.  Sizes: tiny layer; the Flash-Next-shaped layer (2-bit)
# for decode and prefill; the same layer with 3-bit codes; and the 48-layer
# expert stack.
TINY = LayerShape(hidden=256, n_experts=16, top_k=2, inter=64, bits=2, router_bias=False)
FLASH2 = LayerShape(hidden=2560, n_experts=512, top_k=10, inter=640, bits=2, router_bias=True)
FLASH3 = LayerShape(hidden=2560, n_experts=512, top_k=10, inter=640, bits=3, router_bias=True)
# the pruned 256-expert build of the same layer ("Strata Runs 125B
# Qwen3.8-Flash-Next on a 12GB Gaming GPU at Up to 94 Tokens/s", section "The
# Coder build: half the experts, most of the skill"); synthetic weights, and
# how the experts are chosen is not on the path
PRUNED256 = LayerShape(hidden=2560, n_experts=256, top_k=10, inter=640, bits=2,
                       router_bias=True)
# 1-bit codes (w = d (q - 0.5)): the pages mention a 1-bit Coder quant
# ("Open-Source Strata Runs a 125-Billion-Parameter Model ...", Key Facts
# item 4) without a layout; read as the same block-32 family, here on the
# pruned 256-expert Coder shape, and a tiny layer for the oracle's pins
CODER1 = LayerShape(hidden=2560, n_experts=256, top_k=10, inter=640, bits=1, router_bias=True)
TINY1 = LayerShape(hidden=256, n_experts=16, top_k=2, inter=64, bits=1, router_bias=False)
STACK_LAYERS = 48


def _rng(seed: int, layer: int, tensor: int, chunk: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, layer, tensor, chunk])))


def _chunked(n: int, fn, dtype) -> np.ndarray:
    """Fill an array of n elements chunk by chunk (chunk c drawn by fn(c, lo, hi))."""
    out = np.empty(n, dtype=dtype)
    spans = [(c, lo, min(n, lo + _CHUNK)) for c, lo in enumerate(range(0, n, _CHUNK))]

    def work(span):
        c, lo, hi = span
        out[lo:hi] = fn(c, hi - lo)

    workers = min(len(spans), os.cpu_count() or 1, 16)
    if workers <= 1:
        for s in spans:
            work(s)
    else:
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(work, spans))
    return out


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + r) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def hidden(T: int, H: int, seed: int = 0, layer: int = 0) -> np.ndarray:
    """Hidden states [T, H] as bf16 bit patterns, N(0,1)."""
    z = _rng(seed, layer, T_HIDDEN).standard_normal((T, H), dtype=np.float64)
    return f32_to_bf16_bits(z.astype(np.float32))


def router_weight(shape: LayerShape, seed: int = 0, layer: int = 0) -> np.ndarray:
    """Router weight [E, H] fp32, N(0, 1/H) (variance 1/H)."""
    z = _rng(seed, layer, T_ROUTER_W).standard_normal((shape.n_experts, shape.hidden))
    return (z / np.sqrt(shape.hidden)).astype(np.float32)


def router_bias(shape: LayerShape, seed: int = 0, layer: int = 0, s: float = 1.1,
                scale: float = 0.5) -> np.ndarray:
    """Per-expert bias [E] fp32: scale * ln(Zipf(s) pmf of the expert's popularity rank)."""
    E = shape.n_experts
    rank = _rng(seed, layer, T_ROUTER_B).permutation(E) + 1
    pmf_unnorm = np.arange(1, E + 1, dtype=np.float64) ** (-s)
    pmf = pmf_unnorm / pmf_unnorm.sum()
    return (scale * np.log(pmf[rank - 1])).astype(np.float32)


def _codes(n_bytes: int, seed: int, layer: int, tensor: int) -> np.ndarray:
    def draw(c, n):
        words = _rng(seed, layer, tensor, c).bit_generator.random_raw((n + 7) // 8)
        return words.view(np.uint8)[:n]
    return _chunked(n_bytes, draw, np.uint8)


def _scales(n: int, seed: int, layer: int, tensor: int) -> np.ndarray:
    def draw(c, m):
        z = _rng(seed, layer, tensor, c).standard_normal(m, dtype=np.float32)
        d = np.exp(np.float32(np.log(0.02)) + np.float32(0.3) * z)
        return d.astype(np.float16).view(np.uint16)
    return _chunked(n, draw, np.uint16)


@dataclass
class LayerWeights:
    shape: LayerShape
    codes: np.ndarray          # uint8  [E * 3 * mat_code_bytes]
    scales: np.ndarray         # uint16 [E * 3 * mat_scales]
    router_w: np.ndarray       # fp32 [E, H]
    router_b: np.ndarray | None  # fp32 [E]
    shared_codes: np.ndarray   # uint8  [3 * mat_code_bytes]
    shared_scales: np.ndarray  # uint16 [3 * mat_scales]


def layer_weights(shape: LayerShape, seed: int = 0, layer: int = 0) -> LayerWeights:
    E = shape.n_experts
    return LayerWeights(
        shape=shape,
        codes=_codes(E * 3 * shape.mat_code_bytes, seed, layer, T_CODES),
        scales=_scales(E * 3 * shape.mat_scales, seed, layer, T_SCALES),
        router_w=router_weight(shape, seed, layer),
        router_b=router_bias(shape, seed, layer) if shape.router_bias else None,
        shared_codes=_codes(3 * shape.mat_code_bytes, seed, layer, T_SH_CODES),
        shared_scales=_scales(3 * shape.mat_scales, seed, layer, T_SH_SCALES),
    )
