"""Float64 CPU oracle for the fused-QKV projection and grouped-query attention.

TEST INFRASTRUCTURE.  Only the test suite, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA library: it computes the plain definition of each step, in float64,
with no tiling, no online softmax and no split of the key axis.

Sources (page title, then section):

* "Optimize LlamaAttention by fusing QKV projections" (huggingface/transformers
  pull request #40092), the diff of ``LlamaAttention.forward``: one
  ``qkv_proj`` linear layer replaces ``q_proj``/``k_proj``/``v_proj``; its
  output is sliced into query ``[:nh*hd]``, key ``[nh*hd : nh*hd + nkv*hd]``
  and value ``[nh*hd + nkv*hd :]`` features; the review thread notes that
  ``repeat_kv`` later materialises the KV heads for every query head.
* "MHA -> GQA: 提升 LLM 推理效率", section 3.2 (GQA Attention 计算): g query heads
  share one KV head; MHA and MQA are the cases n_kv_heads = n_heads and 1.
* "FlashAttention-3" (together.ai summary), section "FlashAttention方式のおさらい":
  the tiled online-softmax algorithm is exact, so its result equals the plain
  softmax(QK^T)V computed here.
* custom-op overhead gist (``overhead.py``): ``forward(positions,
  hidden_states)`` applies a position-dependent step to q and k only, after
  the fused projection; the attention output (heads concatenated per token)
  then goes through the output projection, and the decoder layer adds the
  residual stream to it.
* "MHA -> GQA: 提升 LLM 推理效率", section 3.2: a PagedAttention KV cache is
  stored non-contiguously, in fixed-size pages that a block table maps to each
  sequence (the paged decode here keeps the tensor cores by making pages whole
  key tiles).
* "FlashAttention-3" (together.ai summary), section "残る最適化と今後の統合":
  the paper adds variable-length sequences.  Read as the packed layout of
  the FlashAttention library: the sequences of a batch are concatenated
  along the token axis and delimited by cumulative offsets (cu_seqlens), so
  that no padding is stored or computed.
* "MHA -> GQA: 提升 LLM 推理效率", section 4.3 (剪枝训练): the new KV projection
  of each group of heads is initialised by mean pooling the group's
  projections (the offline MHA -> GQA weight transform).

Readings where the pages are silent (each restated in the design notes):

* RoPE is the Llama "rotate_half" form: feature i pairs with i + hd/2,
  inv_freq_i = theta^(-2i/hd), x'_i = x_i cos - x_{i+hd/2} sin,
  x'_{i+hd/2} = x_{i+hd/2} cos + x_i sin, angle = position * inv_freq_i.
* softmax scale is 1/sqrt(head_dim).
* query head h reads KV head h // g (contiguous groups, ``repeat_kv``).
* key t is visible to a query at position p iff t < kv_len and, when causal,
  t <= p.  Default query positions are kv_len - S + s (bottom-right aligned).
* a query with no visible key gets an all-zero output row.
* the K/V cache slot of a token is its absolute position.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "fused_projection", "split_qkv", "rope_inv_freq", "apply_rope",
    "qkv_rope_project", "kv_head_of", "softmax", "attend_row",
    "prefill_attention", "decode_attention", "default_q_positions", "round_bf16",
    "varlen_prefill_attention", "output_projection", "meanpool_kv_projection", "gather_pages", "paged_decode_attention",
]


# --------------------------------------------------------------------------
# storage type between calls
# --------------------------------------------------------------------------
def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 value (8 significant bits, ties to even).

    The path stores q, K and V in the call's dtype between calls; chained
    expectations apply this to what one call stores before the next reads it."""
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)                       # a = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


# --------------------------------------------------------------------------
# a1: fused projection; a2 split (pull request #40092, LlamaAttention.forward)
# --------------------------------------------------------------------------
def fused_projection(x: np.ndarray, w_qkv: np.ndarray) -> np.ndarray:
    """Y = X W^T for an ``nn.Linear`` weight stored ``[out_features, in_features]``
    with no bias.  ``x`` is ``[..., hidden]``; returns ``[..., N_qkv]``."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_qkv, dtype=np.float64)
    return x @ w.T


def split_qkv(y: np.ndarray, n_heads: int, n_kv_heads: int, head_dim: int):
    """Slice the fused output into per-head query/key/value features.

    ``y`` is ``[B, S, N_qkv]``; returns q ``[B, S, nh, hd]``, k and v
    ``[B, S, nkv, hd]``.  Within each block, head j owns features
    ``j*hd .. (j+1)*hd - 1``."""
    B, S, N = y.shape
    qn, kn = n_heads * head_dim, n_kv_heads * head_dim
    if N != qn + 2 * kn:
        raise ValueError("fused width does not match (n_heads + 2 n_kv_heads) * head_dim")
    q = y[..., :qn].reshape(B, S, n_heads, head_dim)
    k = y[..., qn:qn + kn].reshape(B, S, n_kv_heads, head_dim)
    v = y[..., qn + kn:].reshape(B, S, n_kv_heads, head_dim)
    return q, k, v


# --------------------------------------------------------------------------
# a2: rotary position embedding (rotate_half pairing; theta from the workload)
# --------------------------------------------------------------------------
def rope_inv_freq(head_dim: int, theta: float) -> np.ndarray:
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * i / head_dim)


def apply_rope(t: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotate ``t`` ``[B, S, H, hd]`` by the angle of each token's position
    ``positions`` ``[B, S]``; pairs are (i, i + hd/2)."""
    t = np.asarray(t, dtype=np.float64)
    hd = t.shape[-1]
    half = hd // 2
    ang = np.asarray(positions, dtype=np.float64)[..., None] * rope_inv_freq(hd, theta)  # [B,S,half]
    c = np.cos(ang)[:, :, None, :]
    s = np.sin(ang)[:, :, None, :]
    lo, hi = t[..., :half], t[..., half:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


def qkv_rope_project(x, w_qkv, positions, n_heads, n_kv_heads, head_dim, theta,
                     k_cache, v_cache):
    """Steps a1-a3: fused projection, RoPE on q and k, scatter.

    Returns ``q`` head-major ``[B, nh, S, hd]`` and copies of the caches
    ``[B, nkv, cap, hd]`` with token s of sequence b written at slot
    ``positions[b, s]``; every other slot keeps its previous value.  Tokens
    whose position lies outside ``[0, cap)`` are not written."""
    y = fused_projection(x, w_qkv)
    q, k, v = split_qkv(y, n_heads, n_kv_heads, head_dim)
    q = apply_rope(q, positions, theta)
    k = apply_rope(k, positions, theta)
    kc = np.array(k_cache, dtype=np.float64, copy=True)
    vc = np.array(v_cache, dtype=np.float64, copy=True)
    B, S = positions.shape
    cap = kc.shape[2]
    for b in range(B):
        for s in range(S):
            p = int(positions[b, s])
            if 0 <= p < cap:
                kc[b, :, p, :] = k[b, s]
                vc[b, :, p, :] = v[b, s]
    return np.ascontiguousarray(q.transpose(0, 2, 1, 3)), kc, vc


# --------------------------------------------------------------------------
# a4-a6: attention (MHA -> GQA blog, section 3.2; FlashAttention recap)
# --------------------------------------------------------------------------
def kv_head_of(h: int, n_heads: int, n_kv_heads: int) -> int:
    """KV head read by query head h: groups of g = nh/nkv consecutive heads."""
    return h // (n_heads // n_kv_heads)


def softmax(scores: np.ndarray) -> np.ndarray:
    """Row softmax with max subtraction; a row of all -inf gives all zeros."""
    s = np.asarray(scores, dtype=np.float64)
    m = np.max(s, axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m)
    z = np.sum(e, axis=-1, keepdims=True)
    return np.divide(e, z, out=np.zeros_like(e), where=z > 0)


def attend_row(q_vec, keys, values, n_visible=None):
    """Plain attention of one query vector over ``keys``/``values`` ``[L, hd]``,
    restricted to the first ``n_visible`` rows; returns (output, probs)."""
    hd = keys.shape[-1]
    L = keys.shape[0] if n_visible is None else int(n_visible)
    if L <= 0:
        return np.zeros(hd), np.zeros(0)
    s = keys[:L] @ np.asarray(q_vec, dtype=np.float64) / np.sqrt(hd)
    p = softmax(s[None, :])[0]
    return p @ values[:L], p


def default_q_positions(kv_lens: np.ndarray, S: int) -> np.ndarray:
    """Bottom-right-aligned positions kv_len - S + s."""
    return (np.asarray(kv_lens, dtype=np.int64)[:, None] - S + np.arange(S)[None, :])


def prefill_attention(q, k_cache, v_cache, kv_lens, causal, q_positions=None,
                      rows=None, chunk=1024):
    """Exact attention for every query row (or the ``rows`` subset).

    q ``[B, nh, S, hd]``; caches ``[B, nkv, cap, hd]``; kv_lens ``[B]``.
    Returns O ``[B, S, nh, hd]`` (when ``rows`` is a list of (b, h, s) triples,
    an array ``[len(rows), hd]`` instead)."""
    q = np.asarray(q, dtype=np.float64)
    kc = np.asarray(k_cache, dtype=np.float64)
    vc = np.asarray(v_cache, dtype=np.float64)
    B, nh, S, hd = q.shape
    nkv = kc.shape[1]
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    pos = default_q_positions(kv_lens, S) if q_positions is None else np.asarray(q_positions, dtype=np.int64)
    scale = 1.0 / np.sqrt(hd)

    def visible_mask(b, s_idx):
        L = int(kv_lens[b])
        t = np.arange(L)[None, :]
        vis = np.ones((len(s_idx), L), dtype=bool)
        if causal:
            vis &= t <= pos[b, s_idx][:, None]
        return vis, L

    if rows is not None:
        out = np.zeros((len(rows), hd))
        for i, (b, h, s) in enumerate(rows):
            j = kv_head_of(h, nh, nkv)
            vis, L = visible_mask(b, np.array([s]))
            if L <= 0:
                continue
            sc = (kc[b, j, :L] @ q[b, h, s]) * scale
            sc = np.where(vis[0], sc, -np.inf)
            p = softmax(sc[None, :])[0]
            out[i] = p @ vc[b, j, :L]
        return out

    out = np.zeros((B, S, nh, hd))
    for b in range(B):
        for h in range(nh):
            j = kv_head_of(h, nh, nkv)
            L = int(kv_lens[b])
            if L <= 0:
                continue
            K, V = kc[b, j, :L], vc[b, j, :L]
            for s0 in range(0, S, chunk):
                s_idx = np.arange(s0, min(S, s0 + chunk))
                vis, _ = visible_mask(b, s_idx)
                sc = (q[b, h, s_idx] @ K.T) * scale
                sc = np.where(vis, sc, -np.inf)
                out[b, s_idx, h] = softmax(sc) @ V
    return out


def decode_attention(q, k_cache, v_cache, kv_lens, pairs=None):
    """One new query per sequence over its cached keys ``[0, kv_len)``.

    q ``[B, nh, hd]``; returns O ``[B, nh, hd]`` (or ``[len(pairs), hd]`` for a
    list of (b, h) pairs).  The split-KV partials and their log-sum-exp merge
    on the GPU reach this same value, because the merge is exact."""
    q = np.asarray(q, dtype=np.float64)
    B, nh, hd = q.shape
    nkv = k_cache.shape[1]
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(nh)]
    out = np.zeros((len(todo), hd))
    for i, (b, h) in enumerate(todo):
        j = kv_head_of(h, nh, nkv)
        L = int(kv_lens[b])
        K = np.asarray(k_cache[b, j, :max(L, 0)], dtype=np.float64)
        V = np.asarray(v_cache[b, j, :max(L, 0)], dtype=np.float64)
        out[i], _ = attend_row(q[b, h], K, V)
    if pairs is None:
        return out.reshape(B, nh, hd)
    return out


def varlen_prefill_attention(q, k, v, cu_seqlens_q, cu_seqlens_k, causal):
    """Prefill attention over packed variable-length sequences.

    q ``[Tq, nh, hd]``, k and v ``[Tk, nkv, hd]``; sequence i owns query rows
    ``[cu_seqlens_q[i], cu_seqlens_q[i+1])`` and key rows
    ``[cu_seqlens_k[i], cu_seqlens_k[i+1])`` and attends to its own keys only.
    With Sq queries over Sk keys, query s of a sequence sits at position
    Sk - Sq + s (bottom-right alignment, as in the padded prefill) and, when
    causal, sees the keys at positions <= its own.  Returns O ``[Tq, nh, hd]``;
    a query that sees no key gets a zero row."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64)
    assert cq.shape == ck.shape and cq[0] == 0 and ck[0] == 0
    assert np.all(np.diff(cq) >= 0) and np.all(np.diff(ck) >= 0)
    Tq, nh, hd = q.shape
    nkv = k.shape[1]
    assert cq[-1] == Tq and ck[-1] == k.shape[0] == v.shape[0]
    out = np.zeros((Tq, nh, hd))
    for i in range(len(cq) - 1):
        Sq, Sk = int(cq[i + 1] - cq[i]), int(ck[i + 1] - ck[i])
        for s in range(Sq):
            n_vis = min(Sk, Sk - Sq + s + 1) if causal else Sk
            for h in range(nh):
                j = kv_head_of(h, nh, nkv)
                keys = k[ck[i]:ck[i + 1], j]
                vals = v[ck[i]:ck[i + 1], j]
                out[cq[i] + s, h], _ = attend_row(q[cq[i] + s, h], keys, vals, max(n_vis, 0))
    return out


def output_projection(attn_out, w_o, residual=None):
    """The attention layer's last step: each token's head outputs
    concatenated in head order (``[..., nh, hd]`` -> ``[..., nh*hd]``) times
    W_o^T (``[hidden, nh*hd]``, nn.Linear layout, no bias), plus the residual
    stream ``[..., hidden]`` when one is given."""
    o = np.asarray(attn_out, dtype=np.float64)
    w = np.asarray(w_o, dtype=np.float64)
    y = o.reshape(o.shape[:-2] + (o.shape[-2] * o.shape[-1],)) @ w.T
    if residual is not None:
        y = y + np.asarray(residual, dtype=np.float64)
    return y


def meanpool_kv_projection(w_qkv_mha: np.ndarray, n_heads: int, n_kv_heads: int,
                           head_dim: int) -> np.ndarray:
    """MHA -> GQA weight transform ("MHA -> GQA" blog, section 4.3): the
    initial projection of each new KV head is the mean of the projections of
    the g = n_heads / n_kv_heads heads of its group; the query projection is
    kept.  The groups are consecutive heads, h -> h // g, the same head map
    as attention uses.

    ``w_qkv_mha`` is the fused MHA weight ``[3 * n_heads * hd, D]`` (query,
    key, value blocks of ``n_heads * hd`` rows each); the result is the fused
    GQA weight ``[(n_heads + 2 * n_kv_heads) * hd, D]``.
    """
    nh, nkv, hd = n_heads, n_kv_heads, head_dim
    assert nh % nkv == 0 and w_qkv_mha.shape[0] == 3 * nh * hd
    g = nh // nkv
    w = np.asarray(w_qkv_mha, dtype=np.float64)
    D = w.shape[1]
    q = w[: nh * hd]
    out = [q]
    for block in (1, 2):                                   # key, then value projection
        heads = w[block * nh * hd:(block + 1) * nh * hd].reshape(nh, hd, D)
        out.append(heads.reshape(nkv, g, hd, D).mean(axis=1).reshape(nkv * hd, D))
    return np.concatenate(out, axis=0)


def gather_pages(pages: np.ndarray, block_table: np.ndarray, kv_lens: np.ndarray, page_size: int) -> np.ndarray:
    """The logical cache ``[B, nkv, cap, hd]`` (cap = pages per sequence x
    page size) of a paged cache: key t of sequence b lives in physical page
    ``block_table[b, t // page_size]`` at row ``t % page_size``; ``pages`` is
    ``[num_pages, nkv, page_size, hd]``.  Rows at or past a sequence's length
    are NaN (never read by attention)."""
    pages = np.asarray(pages, dtype=np.float64)
    B, max_pages = block_table.shape
    _, nkv, ps, hd = pages.shape
    assert ps == page_size
    out = np.full((B, nkv, max_pages * ps, hd), np.nan)
    for b in range(B):
        L = int(kv_lens[b])
        for t in range(0, max(L, 0), ps):
            n = min(ps, L - t)
            out[b, :, t:t + n] = pages[int(block_table[b, t // ps]), :, :n]
    return out


def paged_decode_attention(q, k_pages, v_pages, block_table, kv_lens, page_size, pairs=None):
    """Decode attention over a paged KV cache: the plain decode over the
    logical rows that the block table names."""
    kc = gather_pages(k_pages, block_table, kv_lens, page_size)
    vc = gather_pages(v_pages, block_table, kv_lens, page_size)
    return decode_attention(q, kc, vc, kv_lens, pairs=pairs)

