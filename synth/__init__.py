"""Seeded synthetic inputs for the GQE prefill layer.

This module is shared by the fp64 oracle (``oracle/``) and by the CUDA path's
tests and benchmark. It holds none of the layer's arithmetic: it only draws
numbers. Every tensor is a pure function of ``(seed, stream)``, so both sides
receive identical bits.

Generator (counter based, so any element can be drawn on its own):

* ``splitmix64`` (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): element ``i`` of stream ``s`` under seed ``S`` is
  ``mix(key + (i + 1) * 0x9E3779B97F4A7C15)`` with ``key = mix(S ^ (s * C))``,
  ``C = 0xD1B54A32D192ED03``.
* Two 53-bit uniforms ``u = ((z >> 11) + 1) * 2**-53`` in (0, 1] feed one
  Box-Muller pair ``sqrt(-2 ln u1) * (cos, sin)(2 pi u2)`` (fp64).
* Values are scaled by ``std`` in fp64, rounded to fp32 (round to nearest even),
  and for bf16 tensors rounded again from fp32 to bf16 (round to nearest even).

bf16 tensors are carried as ``uint16`` bit patterns; ``bf16_to_f64`` widens
them exactly.

The workload recipe (x ~ N(0, 1) in bf16, weights ~ N(0, 1/d_model) in bf16,
router weights in fp32, optional skew bias) follows the layer's published
setting: 16 query-head experts in 8 KV groups, head dim 64, k = 1
("Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention",
gist.science summary, Experimental Results).
"""
from __future__ import annotations

import dataclasses
import math
import os

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_STREAM_MUL = np.uint64(0xD1B54A32D192ED03)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

DEFAULT_SEED = 0x6E0E

# One stream id per tensor of a layer instance.
STREAM_X = 1
STREAM_WR = 2
STREAM_WQ = 3
STREAM_WQS = 4
STREAM_WK = 5
STREAM_WV = 6
STREAM_WO = 7
STREAM_WO_DENSE = 8
STREAM_BR = 9


def _mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser, applied in place (z is overwritten and returned)."""
    t = np.empty_like(z)
    np.right_shift(z, np.uint64(30), out=t)
    np.bitwise_xor(z, t, out=z)
    np.multiply(z, _M1, out=z)
    np.right_shift(z, np.uint64(27), out=t)
    np.bitwise_xor(z, t, out=z)
    np.multiply(z, _M2, out=z)
    np.right_shift(z, np.uint64(31), out=t)
    np.bitwise_xor(z, t, out=z)
    return z


def uniform_bits(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    """``n`` raw 64-bit outputs of stream ``stream``, elements ``start..start+n-1``."""
    with np.errstate(over="ignore"):
        key = _mix(np.array([(seed ^ (stream * 0xD1B54A32D192ED03)) & 0xFFFFFFFFFFFFFFFF],
                            dtype=np.uint64))[0]
        z = np.arange(start + 1, start + n + 1, dtype=np.uint64)
        np.multiply(z, _GOLDEN, out=z)
        np.add(z, key, out=z)
        return _mix(z)


def normal_f64(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    """Standard normal fp64 draws ``start..start+n-1`` of a stream.

    Draw ``2i`` and ``2i+1`` are the two halves of one Box-Muller pair made
    from uniforms ``2i`` and ``2i+1``; ``start`` must be even.
    """
    assert start % 2 == 0
    npairs = (n + 1) // 2
    z = uniform_bits(seed, stream, 2 * npairs, start)
    u = ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    th = 2.0 * math.pi * u2
    out = np.empty(2 * npairs, dtype=np.float64)
    out[0::2] = r * np.cos(th)
    out[1::2] = r * np.sin(th)
    return out[:n]


_CHUNK = 1 << 22


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def _bf16_table() -> np.ndarray:
    b = np.arange(65536, dtype=np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


_BF16_F64 = _bf16_table()


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp64 (a bf16 value is the fp32
    value whose upper 16 bits are the pattern; a 65536-entry table holds every
    one of them widened)."""
    return np.take(_BF16_F64, np.ascontiguousarray(bits, dtype=np.uint16))


def bf16_bits_from_f64(a: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (nearest even) -> bf16 (nearest even), as uint16 bits."""
    return f32_to_bf16_bits(np.asarray(a, dtype=np.float64).astype(np.float32))


def normal_bf16(seed: int, stream: int, shape, std: float = 1.0) -> np.ndarray:
    """bf16 bits of N(0, std^2) draws 0..n-1 of a stream. Large tensors are
    drawn in chunks on several threads (numpy releases the GIL in its
    element-wise kernels); every element depends only on its index, so the
    bits do not depend on the chunking."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)

    def fill(s):
        m = min(_CHUNK, n - s)
        out[s:s + m] = bf16_bits_from_f64(normal_f64(seed, stream, m, s) * std)

    starts = range(0, n, _CHUNK)
    if n <= _CHUNK:
        for s in starts:
            fill(s)
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, starts))
    return out.reshape(shape)


def normal_f32(seed: int, stream: int, shape, std: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape))
    return (normal_f64(seed, stream, n) * std).astype(np.float32).reshape(shape)


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Sizes of one GQE layer. Expert ``e = g*M + j`` belongs to KV group ``g``."""
    B: int
    T: int
    d_model: int
    G: int
    M: int
    k: int
    d_head: int

    @property
    def N(self) -> int:
        return self.G * self.M

    @property
    def R(self) -> int:
        return self.B * self.T

    @property
    def n_slots(self) -> int:
        return self.k * self.G + 2


# The workloads the layer is measured on (sizes from the published setting and
# its sequence-length sweep).
TINY = LayerShape(B=1, T=256, d_model=256, G=4, M=2, k=1, d_head=32)
SEQ2K = LayerShape(B=1, T=2048, d_model=1024, G=8, M=2, k=1, d_head=64)
BATCH4_8K = LayerShape(B=4, T=8192, d_model=1024, G=8, M=2, k=1, d_head=64)
SEQ32K = LayerShape(B=1, T=32768, d_model=1024, G=8, M=2, k=1, d_head=64)
SEQ256K = LayerShape(B=1, T=262144, d_model=1024, G=8, M=2, k=1, d_head=64)
SEQ1M = LayerShape(B=1, T=1048576, d_model=1024, G=8, M=2, k=1, d_head=64)
POOL4_K1 = LayerShape(B=1, T=32768, d_model=1024, G=8, M=4, k=1, d_head=64)
POOL4_K2 = LayerShape(B=1, T=32768, d_model=1024, G=8, M=4, k=2, d_head=64)

# Router bias that sends ~80 % of tokens to expert j = 0 of every group when
# logits are iid N(0, 1): P(z0 + beta is among the top k of M) = 0.80.
SKEW_BETA = {(4, 1): 1.8932, (4, 2): 1.0127}


@dataclasses.dataclass
class LayerInputs:
    """One seeded layer instance. bf16 tensors are uint16 bit arrays."""
    shape: LayerShape
    x: np.ndarray          # [R, d] bf16
    W_r: np.ndarray        # [d, N] fp32
    b_r: np.ndarray | None  # [N] fp32 or None
    W_q: np.ndarray        # [d, N*dh] bf16
    W_qs: np.ndarray       # [d, dh] bf16
    W_k: np.ndarray        # [d, G*dh] bf16
    W_v: np.ndarray        # [d, G*dh] bf16
    W_o: np.ndarray        # [(kG+2)*dh, d] bf16
    W_o_dense: np.ndarray  # [N*dh, d] bf16


def make_layer_inputs(shape: LayerShape, seed: int = DEFAULT_SEED, *, skew: bool = False,
                      router_bf16: bool | None = None, with_dense: bool = True) -> LayerInputs:
    """Draw every tensor of one layer instance from ``seed``.

    ``router_bf16`` rounds W_r to bf16 values (held in fp32); by default it is
    on for the tiny d_model=256 layer and off otherwise. ``skew`` adds the
    bias ``SKEW_BETA[(M, k)]`` on expert 0 of each group.
    """
    s = shape
    d, N, dh, G = s.d_model, s.N, s.d_head, s.G
    wstd = 1.0 / math.sqrt(d)
    if router_bf16 is None:
        router_bf16 = d == 256
    x = normal_bf16(seed, STREAM_X, (s.R, d))
    W_r = normal_f32(seed, STREAM_WR, (d, N), wstd)
    if router_bf16:
        W_r = bf16_to_f64(f32_to_bf16_bits(W_r)).astype(np.float32)
    b_r = None
    if skew:
        beta = SKEW_BETA[(s.M, s.k)]
        b_r = np.zeros(N, dtype=np.float32)
        b_r[0::s.M] = np.float32(beta)
    W_q = normal_bf16(seed, STREAM_WQ, (d, N * dh), wstd)
    W_qs = normal_bf16(seed, STREAM_WQS, (d, dh), wstd)
    W_k = normal_bf16(seed, STREAM_WK, (d, G * dh), wstd)
    W_v = normal_bf16(seed, STREAM_WV, (d, G * dh), wstd)
    W_o = normal_bf16(seed, STREAM_WO, (s.n_slots * dh, d), wstd)
    W_o_dense = (normal_bf16(seed, STREAM_WO_DENSE, (N * dh, d), wstd) if with_dense
                 else np.zeros((0, d), dtype=np.uint16))
    return LayerInputs(s, x, W_r, b_r, W_q, W_qs, W_k, W_v, W_o, W_o_dense)
