"""Seeded synthetic inputs for the fused-QKV + grouped-query attention path.

This module is the only code that the float64 oracle and the CUDA library's
callers (tests, bench) share.  It draws random numbers and rounds them to the
storage type; it holds none of the method's arithmetic (no projection, no
rotary embedding, no softmax).

Recipe (every draw is float32 from ``numpy.random.default_rng``; bf16 inputs
are then rounded to nearest-even, and the oracle sees the exact up-cast of
the rounded value, so input rounding is never counted as kernel error):

* hidden states ``x``: N(0, 1)
* fused weight ``W_qkv`` ``[(n_heads + 2 n_kv_heads) * head_dim, hidden]``
  (``nn.Linear`` storage, rows = output features): N(0, 0.02)
* output projection ``W_o`` ``[hidden, n_heads * head_dim]``: N(0, 0.02); the
  residual stream is the layer's own hidden states
* decode queries and KV-cache rows: N(0, 1); cache slots at or beyond a
  sequence's KV length hold NaN, so any read of padding shows in the output
* long-context Q/K/V: N(0, 1) with 0.1 % of the feature channels of each
  tensor multiplied by 20 (the outlier simulation described on the
  FlashAttention-3 page, section "FP8低精度とincoherent processing")
* ragged KV lengths: uniform integers in ``[lo, hi]``

The five workloads are the shapes the pages discuss: a tiny fp32 layer, a
TinyLlama-1.1B-shaped prefill (the model of the fused-QKV pull request), a
Llama-2-7B-shaped batched decode (the model of the MHA -> GQA blog post), the
batch-8 / prompt-16 / 1024-step MQA generation loop of the bigcode multi-query
README, and an 8K-token prefill (the FlashAttention-3 benchmark length).
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

BF16_NAN_BITS = np.uint16(0x7FC0)


# --------------------------------------------------------------------------
# bf16 storage helpers (pure bit manipulation)
# --------------------------------------------------------------------------
def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16, nearest-even; returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    out = r.astype(np.uint16)
    nan = np.isnan(np.ascontiguousarray(a, dtype=np.float32))
    if nan.any():
        out[nan] = BF16_NAN_BITS
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact float32 value of bfloat16 bits."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Tensor:
    """One input tensor: ``store`` is what the GPU receives (uint16 bf16 bits or
    float32), ``f64`` is the exact float64 value the oracle receives."""

    store: np.ndarray
    dtype: str  # "bf16" or "f32"

    @property
    def f64(self) -> np.ndarray:
        if self.dtype == "bf16":
            with np.errstate(invalid="ignore"):          # NaN sentinels in padded caches
                return bf16_to_f32(self.store).astype(np.float64)
        return self.store.astype(np.float64)

    @property
    def shape(self):
        return self.store.shape


def _make(values_f32: np.ndarray, dtype: str) -> Tensor:
    if dtype == "bf16":
        return Tensor(bf16_bits(values_f32), "bf16")
    if dtype == "f32":
        return Tensor(np.ascontiguousarray(values_f32, dtype=np.float32), "f32")
    raise ValueError(dtype)


def _normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


# --------------------------------------------------------------------------
# Workload definitions
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class LayerShape:
    hidden: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    rope_theta: float = 10000.0

    @property
    def n_qkv(self) -> int:
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    dtype: str
    shape: LayerShape
    batch_seq: tuple = ()          # prefill (B, S) cases
    causal: tuple = (True,)
    extra: dict = field(default_factory=dict)


TINY_FP32 = Workload(
    "tiny-gqa-fp32", seed=0, dtype="f32",
    shape=LayerShape(hidden=256, n_heads=8, n_kv_heads=2, head_dim=32),
    batch_seq=((1, 128),), causal=(True,))

TINYLLAMA_PREFILL = Workload(
    "tinyllama-1.1b-prefill", seed=1, dtype="bf16",
    shape=LayerShape(hidden=2048, n_heads=32, n_kv_heads=4, head_dim=64),
    batch_seq=((1, 128), (8, 512), (4, 2048)), causal=(True,))

LLAMA2_DECODE = Workload(
    "llama2-7b-decode", seed=2, dtype="bf16",
    shape=LayerShape(hidden=4096, n_heads=32, n_kv_heads=32, head_dim=128),
    extra=dict(batch=64, kv_lo=512, kv_hi=8192, cap=8192, n_kv_heads_cases=(32, 8, 1)))

MQA_GENERATE = Workload(
    "mqa-generate-b8-p16-g1024", seed=3, dtype="bf16",
    shape=LayerShape(hidden=6144, n_heads=48, n_kv_heads=1, head_dim=128),
    extra=dict(batch=8, prompt=16, steps=1024, cap=1040))

LONG_PREFILL = Workload(
    "long-prefill-8k", seed=4, dtype="bf16",
    shape=LayerShape(hidden=2048, n_heads=16, n_kv_heads=16, head_dim=128),
    batch_seq=((2, 8192),), causal=(True, False),
    extra=dict(n_kv_heads_cases=(16, 4), outlier_frac=0.001, outlier_scale=20.0))

ALL = (TINY_FP32, TINYLLAMA_PREFILL, LLAMA2_DECODE, MQA_GENERATE, LONG_PREFILL)


# --------------------------------------------------------------------------
# Generators
# --------------------------------------------------------------------------
def layer_inputs(shape: LayerShape, B: int, S: int, seed: int, dtype: str,
                 pos_start: int = 0):
    """Hidden states, fused weight and positions for one projection call.

    Draw order: x, then W_qkv.  Positions are ``pos_start .. pos_start+S-1``
    for every sequence (a prompt written from slot ``pos_start`` on)."""
    rng = np.random.default_rng(seed)
    x = _make(_normal(rng, (B, S, shape.hidden)), dtype)
    w = _make(_normal(rng, (shape.n_qkv, shape.hidden), 0.02), dtype)
    pos = np.broadcast_to(np.arange(pos_start, pos_start + S, dtype=np.int32), (B, S)).copy()
    return x, w, pos


def weight(shape: LayerShape, seed: int, dtype: str) -> Tensor:
    rng = np.random.default_rng([seed, 1])
    return _make(_normal(rng, (shape.n_qkv, shape.hidden), 0.02), dtype)


def output_weight(shape: LayerShape, seed: int, dtype: str) -> Tensor:
    """W_o ``[hidden, n_heads * head_dim]`` ~ N(0, 0.02), from its own stream."""
    rng = np.random.default_rng([seed, 8])
    return _make(_normal(rng, (shape.hidden, shape.n_heads * shape.head_dim), 0.02), dtype)


def hidden_states(shape: LayerShape, B: int, S: int, seed: int, stream: int, dtype: str) -> Tensor:
    """x for one call, from its own stream (so step t of a generation loop can be
    regenerated alone)."""
    rng = np.random.default_rng([seed, 2, stream])
    return _make(_normal(rng, (B, S, shape.hidden)), dtype)


def ragged_lengths(B: int, lo: int, hi: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng([seed, 3])
    return rng.integers(lo, hi + 1, size=B).astype(np.int32)


def normal_tensor(shape, seed: int, stream: int, dtype: str, std: float = 1.0) -> Tensor:
    rng = np.random.default_rng([seed, 4, stream])
    return _make(_normal(rng, shape, std), dtype)


def cache_rows(seed: int, tensor_id: int, b: int, j: int, n_rows: int, head_dim: int) -> np.ndarray:
    """float32 N(0,1) rows of one (sequence, KV head) cache slab, from a stream of
    its own so that any slab can be regenerated alone."""
    rng = np.random.default_rng([seed, 5, tensor_id, b, j])
    return _normal(rng, (n_rows, head_dim))


def decode_cache(seed: int, tensor_id: int, B: int, n_kv: int, cap: int, head_dim: int,
                 kv_lens: np.ndarray, dtype: str = "bf16", threads: int = 8) -> Tensor:
    """KV cache ``[B, n_kv, cap, head_dim]``: N(0,1) rows below each sequence's
    KV length, NaN at and beyond it."""
    if dtype == "bf16":
        out = np.full((B, n_kv, cap, head_dim), BF16_NAN_BITS, dtype=np.uint16)
    else:
        out = np.full((B, n_kv, cap, head_dim), np.nan, dtype=np.float32)

    def fill(bj):
        b, j = divmod(bj, n_kv)
        L = int(kv_lens[b])
        rows = cache_rows(seed, tensor_id, b, j, L, head_dim)
        out[b, j, :L] = bf16_bits(rows) if dtype == "bf16" else rows

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fill, range(B * n_kv)))
    return Tensor(out, dtype)


def outlier_channels(n_features: int, frac: float, seed: int, stream: int) -> np.ndarray:
    """Indices of the feature channels (over the flattened heads*head_dim axis)
    that the outlier recipe scales."""
    k = max(1, int(round(frac * n_features)))
    rng = np.random.default_rng([seed, 6, stream])
    return np.sort(rng.choice(n_features, size=k, replace=False))


def outlier_qkv(B: int, S: int, n_heads: int, n_kv: int, head_dim: int, seed: int,
                frac: float = 0.001, scale: float = 20.0, threads: int = 8):
    """Head-major Q ``[B, n_heads, S, hd]`` and K/V ``[B, n_kv, S, hd]`` for the
    long-context prefill: N(0,1) with ``frac`` of each tensor's feature channels
    multiplied by ``scale`` for every token."""
    out = []
    for tid, H in enumerate((n_heads, n_kv, n_kv)):
        vals = np.empty((B, H, S, head_dim), dtype=np.float32)

        def fill(bh, vals=vals, tid=tid, H=H):
            b, h = divmod(bh, H)
            rng = np.random.default_rng([seed, 7, tid, b, h])
            vals[b, h] = rng.standard_normal(size=(S, head_dim), dtype=np.float32)

        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(fill, range(B * H)))
        ch = outlier_channels(H * head_dim, frac, seed, tid)
        for c in ch:
            h, d = divmod(int(c), head_dim)
            vals[:, h, :, d] *= np.float32(scale)
        out.append(_make(vals, "bf16"))
    return tuple(out)
