"""The seeded input recipe (CPU only): the workloads carry the pages' model
shapes, every draw is reproducible, padded cache rows are NaN, and the
outlier recipe scales the stated number of feature channels by the stated
factor for every token."""
import numpy as np
import pytest

import workloads as W


def test_workload_shapes_are_the_pages_models():
    t = W.TINYLLAMA_PREFILL.shape          # TinyLlama-1.1B attention layer
    assert (t.hidden, t.n_heads, t.n_kv_heads, t.head_dim) == (2048, 32, 4, 64)
    assert t.n_qkv == 2560 and W.TINYLLAMA_PREFILL.batch_seq == ((1, 128), (8, 512), (4, 2048))
    d = W.LLAMA2_DECODE                     # Llama-2-7B decode, MHA -> GQA -> MQA caches
    assert (d.shape.hidden, d.shape.n_heads, d.shape.head_dim) == (4096, 32, 128)
    assert d.extra["n_kv_heads_cases"] == (32, 8, 1) and d.extra["batch"] == 64
    assert (d.extra["kv_lo"], d.extra["kv_hi"], d.extra["cap"]) == (512, 8192, 8192)
    g = W.MQA_GENERATE                      # multi-query generation: 48 heads sharing one KV head
    assert (g.shape.hidden, g.shape.n_heads, g.shape.n_kv_heads, g.shape.head_dim) == (6144, 48, 1, 128)
    assert g.shape.n_qkv == 6400
    assert (g.extra["batch"], g.extra["prompt"], g.extra["steps"]) == (8, 16, 1024)
    assert g.extra["cap"] == g.extra["prompt"] + g.extra["steps"]
    lp = W.LONG_PREFILL                     # the 8K-token long-context prefill
    assert lp.batch_seq == ((2, 8192),) and (lp.shape.n_heads, lp.shape.head_dim) == (16, 128)
    assert lp.extra["n_kv_heads_cases"] == (16, 4) and lp.causal == (True, False)
    assert W.TINY_FP32.dtype == "f32" and W.TINY_FP32.shape.n_qkv == 384


def test_draws_are_seeded_and_independent_of_each_other():
    a = W.normal_tensor((3, 5), 9, 0, "bf16")
    np.testing.assert_array_equal(a.store, W.normal_tensor((3, 5), 9, 0, "bf16").store)
    assert not np.array_equal(a.store, W.normal_tensor((3, 5), 9, 1, "bf16").store)
    L = W.ragged_lengths(64, 512, 8192, 2)
    np.testing.assert_array_equal(L, W.ragged_lengths(64, 512, 8192, 2))
    assert L.dtype == np.int32 and L.min() >= 512 and L.max() <= 8192 and len(np.unique(L)) > 32


def test_bf16_inputs_are_exact_bf16_values():
    t = W.normal_tensor((1000,), 3, 0, "bf16")
    f = t.f64.astype(np.float32)
    np.testing.assert_array_equal(W.bf16_bits(f), t.store)           # already representable
    assert np.all((f.view(np.uint32) & 0xFFFF) == 0)


def test_decode_cache_is_nan_beyond_each_length_and_regenerable():
    lens = np.array([0, 1, 7, 16], dtype=np.int32)
    c = W.decode_cache(5, 1, 4, 2, 16, 8, lens)
    v = c.f64
    for b, L in enumerate(lens):
        assert np.all(np.isfinite(v[b, :, :L])) and np.all(np.isnan(v[b, :, L:]))
    # any (sequence, KV head) slab can be drawn again on its own
    np.testing.assert_array_equal(c.store[3, 1, :16], W.bf16_bits(W.cache_rows(5, 1, 3, 1, 16, 8)))
    # the rows of a shorter cache are a prefix of a longer one's
    c2 = W.decode_cache(5, 1, 4, 2, 32, 8, lens * 2)
    np.testing.assert_array_equal(c2.store[2, 0, :7], c.store[2, 0, :7])


@pytest.mark.parametrize("n_features,want", [(2048, 2), (512, 1), (100, 1), (10000, 10)])
def test_outlier_channel_count(n_features, want):
    ch = W.outlier_channels(n_features, 0.001, 4, 0)
    assert len(ch) == want and len(np.unique(ch)) == want and ch.max() < n_features


def test_outlier_recipe_scales_whole_channels_by_twenty():
    B, S, nh, nkv, hd = 1, 512, 16, 4, 128
    q, k, v = W.outlier_qkv(B, S, nh, nkv, hd, seed=4)
    for t, H, tid in ((q, nh, 0), (k, nkv, 1), (v, nkv, 2)):
        x = t.f64.transpose(0, 2, 1, 3).reshape(B * S, H * hd)     # [tokens, features]
        ch = W.outlier_channels(H * hd, 0.001, 4, tid)
        std = x.std(axis=0)
        assert np.all((std[ch] > 15) & (std[ch] < 25))              # x20 for every token
        rest = np.setdiff1d(np.arange(H * hd), ch)
        assert np.all((std[rest] > 0.8) & (std[rest] < 1.25))
