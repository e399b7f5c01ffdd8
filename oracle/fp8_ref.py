"""Float64 CPU oracle for FP8 attention with incoherent processing.

TEST INFRASTRUCTURE.  Only the test suite, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA library.

Source: "FlashAttention-3" (together.ai summary), section "FP8低精度と
incoherent processing": FP8 doubles tensor-core throughput but outliers in
LLM activations inflate the quantisation error; multiplying the queries and
the keys by one random orthogonal matrix spreads the outliers over the
features before quantising, and a Hadamard transform with random signs is
that matrix (cheap, and fusable into the memory-bound step before it, such as
the rotary embedding).  With N(0,1) inputs and 0.1% of the entries made
large, the page reports 2.6x less error than plain FP8 attention.

Readings where the page is silent (each restated in the design notes):

* FP8 format: e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
  largest finite magnitude 448; subnormals down to 2^-9; exponent 15 with
  mantissa 7 is NaN, so there is no infinity).  Rounding to nearest, ties to
  even, saturating at 448.
* Scaling: one scale per tensor, amax / 448, so the largest magnitude maps to
  the largest finite code.
* The rotation acts on the head dimension: Q' = Q M and K' = K M with one M
  for every head of the layer, M = H diag(s) / sqrt(d), H the Sylvester
  Hadamard matrix of order d (a power of two) and s a vector of random signs.
  (Q M)(K M)^T = Q K^T, so without quantisation the scores are unchanged.
* V is quantised as it is (the page rotates only Q and K); P is kept in
  float64 here, so that the comparison isolates the error of the quantised
  Q, K and V.
* The page's 2.6x error reduction comes from a setup it does not state.  With
  per-tensor scales and x20 outliers this oracle measures about 1.4x (per-row
  or per-block scales measured no gain); the pins check the direction.
"""
import numpy as np

E4M3_MAX = 448.0


def sylvester_hadamard(d: int) -> np.ndarray:
    """Unnormalised Hadamard matrix of order d (a power of two):
    H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]."""
    assert d >= 1 and d & (d - 1) == 0, "order must be a power of two"
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def random_sign_hadamard(d: int, signs: np.ndarray) -> np.ndarray:
    """The orthogonal rotation M = H diag(signs) / sqrt(d)."""
    signs = np.asarray(signs, dtype=np.float64)
    assert signs.shape == (d,) and np.all(np.abs(signs) == 1.0)
    return sylvester_hadamard(d) * signs[None, :] / np.sqrt(d)


def e4m3_values() -> np.ndarray:
    """Every finite e4m3 value, decoded from its 8-bit code (NaN codes left
    out), sorted."""
    vals = []
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e, m = (code >> 3) & 0xF, code & 0x7
        if e == 15 and m == 7:
            continue                                   # NaN
        if e == 0:
            v = m / 8.0 * 2.0 ** -6                    # subnormal
        else:
            v = (1.0 + m / 8.0) * 2.0 ** (e - 7)
        vals.append(sign * v)
    return np.unique(np.array(vals))


def round_e4m3(x: np.ndarray) -> np.ndarray:
    """Round to the nearest e4m3 value, ties to the even code, saturating at
    +-448 (the format has no infinity).  Works on the value grid: between two
    neighbouring values a and b, x goes to the nearer one, and at the midpoint
    to the one whose 3-bit mantissa is even."""
    x = np.asarray(x, dtype=np.float64)
    mag = np.minimum(np.abs(x), E4M3_MAX)
    grid = e4m3_values()
    grid = grid[grid >= 0.0]
    idx = np.clip(np.searchsorted(grid, mag), 1, len(grid) - 1)
    lo, hi = grid[idx - 1], grid[idx]
    mid = (lo + hi) / 2.0
    # even mantissa: the code index of a non-negative value counts up by one
    # per grid step from 0, so even grid index = even code = even mantissa
    lo_even = (idx - 1) % 2 == 0
    pick_hi = (mag > mid) | ((mag == mid) & ~lo_even)
    out = np.where(pick_hi, hi, lo)
    out = np.where(mag >= grid[-1], grid[-1], out)
    return np.sign(x) * out


def quantize_e4m3(t: np.ndarray):
    """Per-tensor scaled e4m3 quantisation: returns (dequantised values,
    scale); scale = amax / 448 (1 for an all-zero tensor)."""
    t = np.asarray(t, dtype=np.float64)
    amax = float(np.max(np.abs(t))) if t.size else 0.0
    scale = amax / E4M3_MAX if amax > 0.0 else 1.0
    return round_e4m3(t / scale) * scale, scale


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Non-causal attention ``softmax(q k^T / sqrt(d)) v`` over the last two
    axes (``[..., L, d]``), float64."""
    s = q @ np.swapaxes(k, -1, -2) / np.sqrt(q.shape[-1])
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    return p @ v


def fp8_attention(q, k, v, rotation=None):
    """Attention on e4m3-quantised Q, K and V (each with its own per-tensor
    scale); with ``rotation`` (an orthogonal [d, d] matrix) Q and K are
    multiplied by it first (incoherent processing)."""
    if rotation is not None:
        q = q @ rotation
        k = k @ rotation
    qq, _ = quantize_e4m3(q)
    kq, _ = quantize_e4m3(k)
    vq, _ = quantize_e4m3(v)
    return attention(qq, kq, vq)


def outlier_inputs(shape, frac: float, scale: float, seed: int):
    """The page's experiment: N(0,1) entries, ``frac`` of them multiplied by
    ``scale`` (chosen at random per tensor)."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(3):
        t = rng.standard_normal(shape)
        n = max(1, int(round(frac * t.size)))
        idx = rng.choice(t.size, size=n, replace=False)
        t.flat[idx] *= scale
        out.append(t)
    return out
