"""Pins for the float64 oracle (CPU only).

Nothing here compares the oracle with itself.  Each check ties it to
something the pages or the mathematics fix: the fused-weight slicing printed
in the fused-QKV pull request, the "fused = three separate projections"
equivalence argued there, MHA/MQA as the n_kv_heads extremes of GQA (MHA -> GQA
blog, section 3.2), the exactness of the tiled softmax (FlashAttention-3
summary, recap section) through closed forms and invariants, and literal
brute-force loops on tiny shapes.  The last block plants plausible mistakes in
the oracle and shows that a pin fails for each.
"""
import math
import os

import numpy as np
import pytest

from oracle import gqa_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed=0):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# literal loops (brute force), written independently of the oracle's numpy
# --------------------------------------------------------------------------
def brute_projection(x, w):
    B, S, D = x.shape
    N = w.shape[0]
    y = np.zeros((B, S, N))
    for b in range(B):
        for s in range(S):
            for o in range(N):
                acc = 0.0
                for d in range(D):
                    acc += float(x[b, s, d]) * float(w[o, d])
                y[b, s, o] = acc
    return y


def brute_attention_row(qv, K, V, visible):
    hd = len(qv)
    scores = []
    for t in range(len(K)):
        if visible[t]:
            dot = 0.0
            for d in range(hd):
                dot += qv[d] * K[t][d]
            scores.append((t, dot / math.sqrt(hd)))
    if not scores:
        return [0.0] * hd
    m = max(s for _, s in scores)
    w = [(t, math.exp(s - m)) for t, s in scores]
    z = sum(e for _, e in w)
    out = [0.0] * hd
    for t, e in w:
        for d in range(hd):
            out[d] += e / z * V[t][d]
    return out


# --------------------------------------------------------------------------
# a1 / a2-split
# --------------------------------------------------------------------------
def check_split_matches_page():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "fused_qkv_slices.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) >= 8
    for r in rows:
        nh, nkv, hd, qlo, qhi, klo, khi, vlo, vhi, N = map(int, r)
        y = np.arange(N, dtype=np.float64)[None, None, :]
        q, k, v = ref.split_qkv(y, nh, nkv, hd)
        assert q.shape == (1, 1, nh, hd) and k.shape == (1, 1, nkv, hd) and v.shape == (1, 1, nkv, hd)
        assert q[0, 0, 0, 0] == qlo and q[0, 0, -1, -1] == qhi - 1
        assert k[0, 0, 0, 0] == klo and k[0, 0, -1, -1] == khi - 1
        assert v[0, 0, 0, 0] == vlo and v[0, 0, -1, -1] == vhi - 1
        # head j owns features j*hd .. (j+1)*hd-1 inside each block
        for j in range(nkv):
            assert k[0, 0, j, 0] == klo + j * hd


def test_split_matches_page_slices():
    check_split_matches_page()


def check_fused_equals_separate():
    r = rng(1)
    B, S, D, nh, nkv, hd = 2, 5, 12, 4, 2, 4
    wq = r.standard_normal((nh * hd, D))
    wk = r.standard_normal((nkv * hd, D))
    wv = r.standard_normal((nkv * hd, D))
    x = r.standard_normal((B, S, D))
    w_qkv = np.concatenate([wq, wk, wv], axis=0)          # the pull request's layout
    q, k, v = ref.split_qkv(ref.fused_projection(x, w_qkv), nh, nkv, hd)
    qs = np.einsum("bsd,od->bso", x, wq).reshape(B, S, nh, hd)
    ks = np.einsum("bsd,od->bso", x, wk).reshape(B, S, nkv, hd)
    vs = np.einsum("bsd,od->bso", x, wv).reshape(B, S, nkv, hd)
    np.testing.assert_allclose(q, qs, rtol=0, atol=1e-12)
    np.testing.assert_allclose(k, ks, rtol=0, atol=1e-12)
    np.testing.assert_allclose(v, vs, rtol=0, atol=1e-12)


def test_fused_equals_separate_projections():
    check_fused_equals_separate()


def test_projection_brute_force():
    r = rng(2)
    x = r.standard_normal((2, 3, 7))
    w = r.standard_normal((9, 7))
    np.testing.assert_allclose(ref.fused_projection(x, w), brute_projection(x, w), rtol=0, atol=1e-12)


def test_projection_exact_on_integers():
    # one-hot rows pick weight columns exactly
    D, N = 6, 8
    w = np.arange(N * D, dtype=np.float64).reshape(N, D) - 20
    x = np.eye(D)[None]
    np.testing.assert_array_equal(ref.fused_projection(x, w)[0], w.T)


# --------------------------------------------------------------------------
# a2 RoPE
# --------------------------------------------------------------------------
def test_rope_position_zero_is_identity():
    t = rng(3).standard_normal((2, 4, 3, 16))
    out = ref.apply_rope(t, np.zeros((2, 4), dtype=np.int64), 10000.0)
    np.testing.assert_array_equal(out, t)


def test_rope_preserves_pair_norms():
    t = rng(4).standard_normal((1, 5, 2, 8))
    pos = np.array([[0, 3, 17, 255, 8191]])
    out = ref.apply_rope(t, pos, 10000.0)
    n_in = t[..., :4] ** 2 + t[..., 4:] ** 2
    n_out = out[..., :4] ** 2 + out[..., 4:] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12)


def check_rope_hand_example():
    # hd = 4, theta = 10000: inv_freq = (10000^0, 10000^(-2/4)) = (1, 0.01).
    # Pairs are (0, 2) and (1, 3).  For x = (1, 2, 3, 4):
    #   position 1: pair (0,2) turns by 1 rad, pair (1,3) by 0.01 rad
    #   position 2: by 2 rad and 0.02 rad
    x = np.array([1.0, 2.0, 3.0, 4.0])
    for p, (a0, a1) in ((1, (1.0, 0.01)), (2, (2.0, 0.02))):
        want = np.array([
            1 * math.cos(a0) - 3 * math.sin(a0),
            2 * math.cos(a1) - 4 * math.sin(a1),
            3 * math.cos(a0) + 1 * math.sin(a0),
            4 * math.cos(a1) + 2 * math.sin(a1),
        ])
        got = ref.apply_rope(x[None, None, None, :], np.array([[p]]), 10000.0)[0, 0, 0]
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)


def test_rope_hand_example():
    check_rope_hand_example()


def test_rope_pairing_plane_and_angle():
    # A vector with only feature i set stays in span{e_i, e_(i+hd/2)} and turns
    # by position * theta^(-2i/hd).
    hd, theta = 16, 10000.0
    for i in range(hd // 2):
        e = np.zeros(hd)
        e[i] = 1.0
        out = ref.apply_rope(e[None, None, None], np.array([[5]]), theta)[0, 0, 0]
        others = np.delete(out, [i, i + hd // 2])
        assert np.all(others == 0.0)
        ang = math.atan2(out[i + hd // 2], out[i])
        want = 5 * theta ** (-2 * i / hd)
        want = math.atan2(math.sin(want), math.cos(want))
        assert abs(ang - want) < 1e-12


def test_rope_relative_position_property():
    # q(p+c) . k(p'+c) == q(p) . k(p') for every shift c
    r = rng(5)
    q = r.standard_normal((1, 1, 1, 32))
    k = r.standard_normal((1, 1, 1, 32))
    base = None
    for c in (0, 1, 7, 100, 4000):
        qq = ref.apply_rope(q, np.array([[12 + c]]), 10000.0)
        kk = ref.apply_rope(k, np.array([[3 + c]]), 10000.0)
        d = float(np.sum(qq * kk))
        base = d if base is None else base
        assert abs(d - base) < 1e-9


def test_rope_composes():
    t = rng(6).standard_normal((1, 1, 1, 8))
    a = ref.apply_rope(ref.apply_rope(t, np.array([[3]]), 500.0), np.array([[4]]), 500.0)
    b = ref.apply_rope(t, np.array([[7]]), 500.0)
    np.testing.assert_allclose(a, b, atol=1e-13)


# --------------------------------------------------------------------------
# a3 scatter into the head-major cache
# --------------------------------------------------------------------------
def test_scatter_slots_and_sentinels():
    B, S, D, nh, nkv, hd, cap = 2, 3, 8, 4, 2, 4, 10
    w = (np.arange((nh + 2 * nkv) * hd * D).reshape(-1, D) % 7) - 3.0
    x = np.zeros((B, S, D))
    for b in range(B):
        for s in range(S):
            x[b, s, (b * S + s) % D] = 1.0
    pos = np.array([[0, 4, 9], [2, 3, 12]])        # 12 >= cap: not written
    sentinel = -12345.0
    kc0 = np.full((B, nkv, cap, hd), sentinel)
    vc0 = np.full((B, nkv, cap, hd), sentinel)
    q, kc, vc = ref.qkv_rope_project(x, w, pos, nh, nkv, hd, 10000.0, kc0, vc0)
    assert q.shape == (B, nh, S, hd)
    written = {(b, int(p)) for b in range(B) for p in pos[b] if p < cap}
    for b in range(B):
        for slot in range(cap):
            if (b, slot) not in written:
                assert np.all(kc[b, :, slot] == sentinel) and np.all(vc[b, :, slot] == sentinel)
    # V has no rotation: exact copy of the projected integers at slot = position
    for b in range(B):
        for s in range(S):
            p = int(pos[b, s])
            if p >= cap:
                continue
            col = (b * S + s) % D
            v_feat = w[(nh + nkv) * hd:, col].reshape(nkv, hd)
            np.testing.assert_array_equal(vc[b, :, p], v_feat)
            if p == 0:  # rotation by zero: K and Q exact too
                np.testing.assert_array_equal(kc[b, :, p], w[nh * hd:(nh + nkv) * hd, col].reshape(nkv, hd))
                np.testing.assert_array_equal(q[b, :, s], w[:nh * hd, col].reshape(nh, hd))


# --------------------------------------------------------------------------
# a4-a6 attention
# --------------------------------------------------------------------------
def _rand_attn(r, B, nh, nkv, S, L, hd, cap=None):
    cap = cap or L
    q = r.standard_normal((B, nh, S, hd))
    kc = r.standard_normal((B, nkv, cap, hd))
    vc = r.standard_normal((B, nkv, cap, hd))
    return q, kc, vc


def test_softmax_rows_sum_to_one():
    s = rng(7).standard_normal((50, 33)) * 30
    p = ref.softmax(s)
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-13)
    # invariance to a constant shift per row
    np.testing.assert_allclose(ref.softmax(s + 1e3), p, atol=1e-13)


def check_closed_form_two_keys():
    # hd = 4: q = (2,0,0,0), k0 = (1,0,0,0), k1 = 0 -> scores (2/sqrt(4), 0) = (1, 0)
    # so p0 = e/(1+e), p1 = 1/(1+e) and O = p0 v0 + p1 v1.
    q = np.array([2.0, 0, 0, 0])
    K = np.array([[1.0, 0, 0, 0], [0, 0, 0, 0]])
    V = np.array([[1.0, 2, 3, 4], [-1.0, 0, 5, 1]])
    p0 = math.e / (1 + math.e)
    want = p0 * V[0] + (1 - p0) * V[1]
    out, p = ref.attend_row(q, K, V)
    np.testing.assert_allclose(p, [p0, 1 - p0], atol=1e-15)
    np.testing.assert_allclose(out, want, atol=1e-15)
    # the same through the batched prefill / decode entry points
    qq = q.reshape(1, 1, 1, 4)
    kc, vc = K.reshape(1, 1, 2, 4), V.reshape(1, 1, 2, 4)
    o = ref.prefill_attention(qq, kc, vc, np.array([2]), causal=False)
    np.testing.assert_allclose(o[0, 0, 0], want, atol=1e-15)
    o = ref.decode_attention(qq[:, :, 0], kc, vc, np.array([2]))
    np.testing.assert_allclose(o[0, 0], want, atol=1e-15)


def test_closed_form_two_keys():
    check_closed_form_two_keys()


def test_identical_keys_give_mean_of_visible_values():
    r = rng(8)
    B, nh, nkv, S, hd = 2, 4, 2, 6, 8
    q = r.standard_normal((B, nh, S, hd))
    k_row = r.standard_normal(hd)
    kc = np.broadcast_to(k_row, (B, nkv, S, hd)).copy()
    vc = r.standard_normal((B, nkv, S, hd))
    lens = np.array([S, S])
    o = ref.prefill_attention(q, kc, vc, lens, causal=False)
    for b in range(B):
        for h in range(nh):
            j = h // (nh // nkv)
            np.testing.assert_allclose(o[b, :, h], np.broadcast_to(vc[b, j].mean(0), (S, hd)), atol=1e-13)
    o = ref.prefill_attention(q, kc, vc, lens, causal=True)
    for i in range(S):
        np.testing.assert_allclose(o[1, i, 3], vc[1, 1, :i + 1].mean(0), atol=1e-13)
    # q = 0 gives uniform weights whatever the keys are
    kc2 = r.standard_normal((B, nkv, S, hd))
    o = ref.prefill_attention(np.zeros_like(q), kc2, vc, lens, causal=True)
    np.testing.assert_allclose(o[0, 4, 0], vc[0, 0, :5].mean(0), atol=1e-13)


def test_single_visible_key_returns_its_value():
    r = rng(9)
    q, kc, vc = _rand_attn(r, 1, 2, 1, 5, 5, 8)
    o = ref.prefill_attention(q, kc, vc, np.array([5]), causal=True)
    np.testing.assert_allclose(o[0, 0, 0], vc[0, 0, 0], atol=1e-15)
    np.testing.assert_allclose(o[0, 0, 1], vc[0, 0, 0], atol=1e-15)


def test_no_visible_key_gives_zero_row():
    r = rng(10)
    q, kc, vc = _rand_attn(r, 1, 2, 1, 3, 4, 8)
    o = ref.prefill_attention(q, kc, vc, np.array([0]), causal=True)
    assert np.all(o == 0)
    o = ref.decode_attention(q[:, :, 0], kc, vc, np.array([0]))
    assert np.all(o == 0)


def test_noncausal_permutation_invariance():
    r = rng(11)
    q, kc, vc = _rand_attn(r, 1, 4, 2, 3, 9, 8)
    perm = r.permutation(9)
    o1 = ref.prefill_attention(q, kc, vc, np.array([9]), causal=False)
    o2 = ref.prefill_attention(q, kc[:, :, perm], vc[:, :, perm], np.array([9]), causal=False)
    np.testing.assert_allclose(o1, o2, atol=1e-13)


def check_gqa_equals_mha_with_repeated_kv():
    r = rng(12)
    B, nh, S, hd = 2, 8, 5, 8
    for nkv in (1, 2, 4, 8):
        q, kc, vc = _rand_attn(r, B, nh, nkv, S, S, hd)
        lens = np.array([S, S - 2])
        g = nh // nkv
        kr, vr = np.repeat(kc, g, axis=1), np.repeat(vc, g, axis=1)   # repeat_kv
        for causal in (True, False):
            np.testing.assert_allclose(
                ref.prefill_attention(q, kc, vc, lens, causal),
                ref.prefill_attention(q, kr, vr, lens, causal), atol=1e-13)
        np.testing.assert_allclose(
            ref.decode_attention(q[:, :, -1], kc, vc, lens),
            ref.decode_attention(q[:, :, -1], kr, vr, lens), atol=1e-13)


def test_gqa_equals_mha_with_repeated_kv():
    check_gqa_equals_mha_with_repeated_kv()


def test_mqa_every_head_reads_the_single_kv_head():
    r = rng(13)
    q, kc, vc = _rand_attn(r, 1, 6, 1, 4, 4, 8)
    o = ref.prefill_attention(q, kc, vc, np.array([4]), causal=False)
    for h in range(6):
        oh = ref.prefill_attention(q[:, h:h + 1], kc, vc, np.array([4]), causal=False)
        np.testing.assert_allclose(o[:, :, h], oh[:, :, 0], atol=1e-14)


def check_last_causal_row_equals_decode():
    r = rng(14)
    B, nh, nkv, S, hd = 2, 4, 2, 7, 16
    q, kc, vc = _rand_attn(r, B, nh, nkv, S, S, hd)
    lens = np.array([S, S])
    o = ref.prefill_attention(q, kc, vc, lens, causal=True)
    d = ref.decode_attention(q[:, :, -1], kc, vc, lens)
    np.testing.assert_allclose(o[:, -1], d, atol=1e-13)
    # and every causal row s equals a decode with kv_len = s + 1
    for s in range(S):
        d = ref.decode_attention(q[:, :, s], kc, vc, np.array([s + 1, s + 1]))
        np.testing.assert_allclose(o[:, s], d, atol=1e-13)


def test_last_causal_prefill_row_equals_decode_step():
    check_last_causal_row_equals_decode()


def test_bottom_right_causal_alignment_and_explicit_positions():
    r = rng(15)
    B, nh, nkv, S, L, hd = 1, 2, 1, 3, 10, 8
    q, kc, vc = _rand_attn(r, B, nh, nkv, S, L, hd)
    lens = np.array([L])
    o = ref.prefill_attention(q, kc, vc, lens, causal=True)
    for s in range(S):   # query s sits at position L - S + s and sees keys 0..L-S+s
        want, _ = ref.attend_row(q[0, 1, s], kc[0, 0], vc[0, 0], L - S + s + 1)
        np.testing.assert_allclose(o[0, s, 1], want, atol=1e-13)
    o2 = ref.prefill_attention(q, kc, vc, lens, causal=True, q_positions=np.array([[7, 8, 9]]))
    np.testing.assert_allclose(o, o2, atol=0)


def test_nan_padding_never_reaches_output():
    r = rng(16)
    q, kc, vc = _rand_attn(r, 2, 4, 2, 3, 12, 8)
    lens = np.array([5, 12])
    kc[0, :, 5:] = np.nan
    vc[0, :, 5:] = np.nan
    o = ref.prefill_attention(q, kc, vc, lens, causal=False)
    d = ref.decode_attention(q[:, :, 0], kc, vc, lens)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(d))


def check_brute_force_attention():
    r = rng(17)
    for (B, nh, nkv, S, L, hd) in ((1, 2, 1, 3, 5, 4), (2, 4, 2, 6, 6, 8), (2, 4, 1, 4, 6, 2)):
        q, kc, vc = _rand_attn(r, B, nh, nkv, S, L, hd)
        lens = np.array([L - 1, L][:B])
        for causal in (True, False):
            o = ref.prefill_attention(q, kc, vc, lens, causal)
            for b in range(B):
                for h in range(nh):
                    j = h * nkv // nh
                    for s in range(S):
                        p = lens[b] - S + s
                        vis = [t < lens[b] and (not causal or t <= p) for t in range(L)]
                        want = brute_attention_row(list(q[b, h, s]), kc[b, j].tolist(), vc[b, j].tolist(), vis)
                        np.testing.assert_allclose(o[b, s, h], want, rtol=0, atol=1e-12)
        d = ref.decode_attention(q[:, :, 0], kc, vc, lens)
        for b in range(B):
            for h in range(nh):
                j = h * nkv // nh
                vis = [t < lens[b] for t in range(L)]
                want = brute_attention_row(list(q[b, h, 0]), kc[b, j].tolist(), vc[b, j].tolist(), vis)
                np.testing.assert_allclose(d[b, h], want, rtol=0, atol=1e-12)


def test_brute_force_attention():
    check_brute_force_attention()


def test_generation_loop_equals_causal_prefill():
    """Prompt prefill then one-token decode steps that grow the cache in place
    give the rows of one causal prefill over all tokens."""
    r = rng(18)
    B, D, nh, nkv, hd, P, T = 2, 16, 4, 1, 8, 3, 4
    cap = P + T
    w = r.standard_normal(((nh + 2 * nkv) * hd, D)) * 0.3
    x = r.standard_normal((B, P + T, D))
    pos = np.broadcast_to(np.arange(P + T), (B, P + T))
    kc0 = np.full((B, nkv, cap, hd), np.nan)
    vc0 = np.full((B, nkv, cap, hd), np.nan)
    q_all, kc_all, vc_all = ref.qkv_rope_project(x, w, pos, nh, nkv, hd, 10000.0, kc0, vc0)
    full = ref.prefill_attention(q_all, kc_all, vc_all, np.array([cap, cap]), causal=True)
    q_p, kc, vc = ref.qkv_rope_project(x[:, :P], w, pos[:, :P], nh, nkv, hd, 10000.0, kc0, vc0)
    o_p = ref.prefill_attention(q_p, kc, vc, np.array([P, P]), causal=True)
    np.testing.assert_allclose(o_p, full[:, :P], atol=1e-12)
    for t in range(T):
        q_t, kc, vc = ref.qkv_rope_project(x[:, P + t:P + t + 1], w, pos[:, P + t:P + t + 1],
                                           nh, nkv, hd, 10000.0, kc, vc)
        o_t = ref.decode_attention(q_t[:, :, 0], kc, vc, np.array([P + t + 1] * B))
        np.testing.assert_allclose(o_t, full[:, P + t], atol=1e-12)


# --------------------------------------------------------------------------
# planted mistakes: each must make at least one pin fail
# --------------------------------------------------------------------------
def _fails(check):
    try:
        check()
    except AssertionError:
        return True
    return False


def test_planted_wrong_head_map_is_caught(monkeypatch):
    monkeypatch.setattr(ref, "kv_head_of", lambda h, nh, nkv: h % nkv)
    assert _fails(check_gqa_equals_mha_with_repeated_kv)
    assert _fails(check_brute_force_attention)


def test_planted_dropped_scale_is_caught(monkeypatch):
    orig = ref.softmax
    monkeypatch.setattr(ref, "np", _NumpyNoSqrt())
    assert _fails(check_closed_form_two_keys)
    monkeypatch.setattr(ref, "softmax", orig)


class _NumpyNoSqrt:
    """numpy with sqrt replaced by 1 (drops the 1/sqrt(hd) softmax scale)."""

    def __getattr__(self, name):
        if name == "sqrt":
            return lambda x: 1.0
        return getattr(np, name)


def test_planted_interleaved_rope_is_caught(monkeypatch):
    def interleaved(t, positions, theta):
        t = np.asarray(t, dtype=np.float64)
        hd = t.shape[-1]
        ang = np.asarray(positions, dtype=np.float64)[..., None] * ref.rope_inv_freq(hd, theta)
        c, s = np.cos(ang)[:, :, None, :], np.sin(ang)[:, :, None, :]
        ev, od = t[..., 0::2], t[..., 1::2]
        out = np.empty_like(t)
        out[..., 0::2] = ev * c - od * s
        out[..., 1::2] = od * c + ev * s
        return out
    monkeypatch.setattr(ref, "apply_rope", interleaved)
    assert _fails(check_rope_hand_example)


def test_planted_rope_sign_error_is_caught(monkeypatch):
    orig = ref.apply_rope
    monkeypatch.setattr(ref, "apply_rope", lambda t, p, th: orig(t, -np.asarray(p), th))
    assert _fails(check_rope_hand_example)


def test_planted_swapped_kv_slices_is_caught(monkeypatch):
    orig = ref.split_qkv

    def swapped(y, nh, nkv, hd):
        q, k, v = orig(y, nh, nkv, hd)
        return q, v, k
    monkeypatch.setattr(ref, "split_qkv", swapped)
    assert _fails(check_split_matches_page)
    assert _fails(check_fused_equals_separate)


def test_planted_transposed_weight_is_caught(monkeypatch):
    monkeypatch.setattr(ref, "fused_projection",
                        lambda x, w: np.asarray(x) @ np.asarray(w).reshape(w.shape[1], w.shape[0]))
    assert _fails(check_fused_equals_separate)


def test_planted_off_by_one_causal_is_caught(monkeypatch):
    orig = ref.default_q_positions
    monkeypatch.setattr(ref, "default_q_positions", lambda kv, S: orig(kv, S) - 1)
    assert _fails(check_last_causal_row_equals_decode)


# --------------------------------------------------------------------------
# bf16 storage rounding used for chained expectations
# --------------------------------------------------------------------------
def test_round_bf16_matches_bit_level_rounding():
    """Independent route: float32 bits rounded to nearest-even in the input
    module (integer arithmetic) versus frexp/rint here."""
    import workloads as W
    r = rng(30)
    a = np.concatenate([r.standard_normal(200000), r.standard_normal(1000) * 1e4,
                        r.standard_normal(1000) * 1e-4]).astype(np.float32)
    want = W.bf16_to_f32(W.bf16_bits(a)).astype(np.float64)
    np.testing.assert_array_equal(ref.round_bf16(a.astype(np.float64)), want)


def test_round_bf16_matches_the_library_cast():
    """A third route: torch's float32 -> bfloat16 cast (nearest, ties to even),
    on random values and on exact midpoints between neighbouring bf16 values."""
    import torch
    r = rng(32)
    a = np.concatenate([r.standard_normal(100000) * 3, r.standard_normal(1000) * 1e-30]).astype(np.float32)
    mids = (a.view(np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)    # halfway bit patterns
    a = np.concatenate([a, mids.view(np.float32)])
    lib = torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ref.round_bf16(a.astype(np.float64)), lib)


def test_round_bf16_exact_and_ties_to_even():
    exact = np.array([1.0, -2.0, 1.5, 0.00390625, 3.0 * 2 ** 40, 1 + 2 ** -7])
    np.testing.assert_array_equal(ref.round_bf16(exact), exact)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1.0)
    assert ref.round_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    assert ref.round_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6
    a = rng(31).standard_normal(10000) * 37
    assert np.max(np.abs(ref.round_bf16(a) - a) / np.abs(a)) <= 2 ** -8


# --------------------------------------------------------------------------
# MHA -> GQA weight transform (MHA -> GQA blog, section 4.3: mean pooling of
# each group's projections)
# --------------------------------------------------------------------------
def brute_meanpool(w, nh, nkv, hd):
    g = nh // nkv
    D = w.shape[1]
    out = np.zeros(((nh + 2 * nkv) * hd, D))
    for r in range(nh * hd):
        out[r] = w[r]
    for block in (1, 2):
        for j in range(nkv):
            for d in range(hd):
                for c in range(D):
                    acc = 0.0
                    for i in range(g):
                        acc += float(w[block * nh * hd + (j * g + i) * hd + d, c])
                    out[nh * hd + (block - 1) * nkv * hd + j * hd + d, c] = acc / g
    return out


def check_meanpool_of_equal_heads_turns_mha_into_gqa():
    """A GQA weight whose KV heads are replicated g times (consecutive heads,
    as repeat_kv does) is an MHA weight with equal heads in each group.
    Pooling it gives the GQA weight back, and the layer computes the same
    attention as MHA before the transform and as GQA after it."""
    nh, nkv, hd, D, B, S = 4, 2, 4, 8, 1, 5
    g = nh // nkv
    r = rng(41)
    w_gqa = r.normal(size=((nh + 2 * nkv) * hd, D))
    kv = [w_gqa[nh * hd + k * nkv * hd: nh * hd + (k + 1) * nkv * hd].reshape(nkv, hd, D) for k in (0, 1)]
    w_mha = np.concatenate([w_gqa[: nh * hd]] + [np.repeat(t, g, axis=0).reshape(nh * hd, D) for t in kv])
    pooled = ref.meanpool_kv_projection(w_mha, nh, nkv, hd)
    np.testing.assert_allclose(pooled, w_gqa, rtol=0, atol=1e-12)
    x = r.normal(size=(B, S, D))
    pos = np.arange(S)[None, :]
    lens = np.array([S])
    outs = []
    for w, kvh in ((w_mha, nh), (pooled, nkv)):
        q, kc, vc = ref.qkv_rope_project(x, w, pos, nh, kvh, hd, 10000.0,
                                         np.zeros((B, kvh, S, hd)), np.zeros((B, kvh, S, hd)))
        outs.append(ref.prefill_attention(q, kc, vc, lens, True))
    np.testing.assert_allclose(outs[0], outs[1], rtol=0, atol=1e-12)


def test_meanpool_of_equal_heads_turns_mha_into_gqa():
    check_meanpool_of_equal_heads_turns_mha_into_gqa()


def test_meanpool_brute_force():
    nh, nkv, hd, D = 6, 2, 2, 3
    w = rng(42).normal(size=(3 * nh * hd, D))
    np.testing.assert_allclose(ref.meanpool_kv_projection(w, nh, nkv, hd), brute_meanpool(w, nh, nkv, hd),
                               rtol=0, atol=1e-12)


def test_meanpool_mha_is_identity_and_mqa_averages_every_head():
    nh, hd, D = 4, 2, 5
    w = rng(43).normal(size=(3 * nh * hd, D))
    np.testing.assert_array_equal(ref.meanpool_kv_projection(w, nh, nh, hd), w)     # n_kv_heads = n_heads
    mqa = ref.meanpool_kv_projection(w, nh, 1, hd)                                   # n_kv_heads = 1
    assert mqa.shape == ((nh + 2) * hd, D)
    for block in (1, 2):
        heads = [w[block * nh * hd + h * hd: block * nh * hd + (h + 1) * hd] for h in range(nh)]
        want = sum(heads) / nh
        np.testing.assert_allclose(mqa[nh * hd + (block - 1) * hd: nh * hd + block * hd], want, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(mqa[: nh * hd], w[: nh * hd])                       # query rows kept


def test_meanpool_is_linear():
    nh, nkv, hd, D = 8, 2, 4, 3
    r = rng(44)
    a, b = r.normal(size=(3 * nh * hd, D)), r.normal(size=(3 * nh * hd, D))
    lhs = ref.meanpool_kv_projection(2.0 * a - 0.5 * b, nh, nkv, hd)
    rhs = 2.0 * ref.meanpool_kv_projection(a, nh, nkv, hd) - 0.5 * ref.meanpool_kv_projection(b, nh, nkv, hd)
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-12)


def test_planted_strided_pooling_groups_are_caught(monkeypatch):
    """Pooling heads h with the same h mod nkv (instead of the consecutive
    groups h // g that attention reads) breaks the MHA -> GQA identity."""
    def strided(w, nh, nkv, hd):
        D = w.shape[1]
        out = [w[: nh * hd]]
        for block in (1, 2):
            heads = w[block * nh * hd:(block + 1) * nh * hd].reshape(nh // nkv, nkv, hd, D)
            out.append(heads.mean(axis=0).reshape(nkv * hd, D))
        return np.concatenate(out)
    monkeypatch.setattr(ref, "meanpool_kv_projection", strided)
    assert _fails(check_meanpool_of_equal_heads_turns_mha_into_gqa)


# --------------------------------------------------------------------------
# paged KV cache (MHA -> GQA blog, section 3.2: PagedAttention's
# non-contiguous cache)
# --------------------------------------------------------------------------
def paged_setup(seed=51, B=3, nkv=2, nh=4, hd=4, ps=4, max_pages=3):
    r = rng(seed)
    cap = ps * max_pages
    kc, vc = r.normal(size=(B, nkv, cap, hd)), r.normal(size=(B, nkv, cap, hd))
    q = r.normal(size=(B, nh, hd))
    lens = np.array([cap, 5, 1])[:B]
    # the contiguous cache cut into pages: page (b, p) = rows [p*ps, (p+1)*ps) of sequence b
    kp = kc.reshape(B, nkv, max_pages, ps, hd).transpose(0, 2, 1, 3, 4).reshape(B * max_pages, nkv, ps, hd)
    vp = vc.reshape(B, nkv, max_pages, ps, hd).transpose(0, 2, 1, 3, 4).reshape(B * max_pages, nkv, ps, hd)
    table = np.arange(B * max_pages).reshape(B, max_pages)
    return q, kc, vc, kp, vp, table, lens, ps


def check_paged_page_order_does_not_matter():
    q, kc, vc, kp, vp, table, lens, ps = paged_setup()
    base = ref.paged_decode_attention(q, kp, vp, table, lens, ps)
    perm = rng(52).permutation(kp.shape[0])            # physical page i moves to slot perm[i]
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    np.testing.assert_array_equal(ref.paged_decode_attention(q, kp2, vp2, perm[table], lens, ps), base)


def test_paged_cache_with_identity_table_is_the_contiguous_cache():
    q, kc, vc, kp, vp, table, lens, ps = paged_setup()
    g = ref.gather_pages(kp, table, lens, ps)
    for b, L in enumerate(lens):
        np.testing.assert_array_equal(g[b, :, :L], kc[b, :, :L])
        assert np.all(np.isnan(g[b, :, L:]))
    np.testing.assert_array_equal(ref.paged_decode_attention(q, kp, vp, table, lens, ps),
                                  ref.decode_attention(q, kc, vc, lens))


def test_paged_page_order_does_not_matter():
    check_paged_page_order_does_not_matter()


def test_paged_brute_force():
    q, kc, vc, kp, vp, table, lens, ps = paged_setup(seed=53)
    perm = rng(54).permutation(kp.shape[0])
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    t2 = perm[table]
    B, nh, hd = q.shape
    nkv = kp.shape[1]
    want = np.zeros((B, nh, hd))
    for b in range(B):
        for h in range(nh):
            j = h // (nh // nkv)
            scores, vals = [], []
            for t in range(int(lens[b])):
                page, row = int(t2[b, t // ps]), t % ps
                scores.append(sum(float(q[b, h, d]) * float(kp2[page, j, row, d]) for d in range(hd)) / math.sqrt(hd))
                vals.append(vp2[page, j, row])
            m = max(scores)
            w = [math.exp(s_ - m) for s_ in scores]
            want[b, h] = sum(wi * vi for wi, vi in zip(w, vals)) / sum(w)
    np.testing.assert_allclose(ref.paged_decode_attention(q, kp2, vp2, t2, lens, ps), want, rtol=0, atol=1e-12)


def test_planted_ignored_block_table_is_caught(monkeypatch):
    """Reading page p of sequence b from physical page b*max_pages + p (the
    table ignored) breaks the page-order invariance."""
    orig = ref.gather_pages

    def ignore_table(pages, block_table, kv_lens, page_size):
        B, max_pages = block_table.shape
        return orig(pages, np.arange(B * max_pages).reshape(B, max_pages), kv_lens, page_size)
    monkeypatch.setattr(ref, "gather_pages", ignore_table)
    assert _fails(check_paged_page_order_does_not_matter)



# --------------------------------------------------------------------------
# packed variable-length prefill (FlashAttention-3 summary, section
# "残る最適化と今後の統合": variable-length sequences; cu_seqlens offsets)
# --------------------------------------------------------------------------
def varlen_setup(seed=61, nh=4, nkv=2, hd=4, q_lens=(3, 0, 5, 1, 4), k_lens=(5, 2, 5, 1, 9)):
    r = rng(seed)
    cq = np.concatenate([[0], np.cumsum(q_lens)])
    ck = np.concatenate([[0], np.cumsum(k_lens)])
    q = r.normal(size=(cq[-1], nh, hd))
    k = r.normal(size=(ck[-1], nkv, hd))
    v = r.normal(size=(ck[-1], nkv, hd))
    return q, k, v, cq, ck


def brute_varlen(q, k, v, cq, ck, causal):
    """Literal loops: for each packed query row, find its sequence by
    scanning the offsets, then softmax over that sequence's visible keys."""
    Tq, nh, hd = q.shape
    nkv = k.shape[1]
    out = np.zeros((Tq, nh, hd))
    for r_ in range(Tq):
        i = max(n for n in range(len(cq) - 1) if cq[n] <= r_ < cq[n + 1])
        Sq, Sk = cq[i + 1] - cq[i], ck[i + 1] - ck[i]
        pos = Sk - Sq + (r_ - cq[i])
        for h in range(nh):
            j = h // (nh // nkv)
            keys = [t for t in range(Sk) if not causal or t <= pos]
            if not keys:
                continue
            sc = [sum(float(q[r_, h, d]) * float(k[ck[i] + t, j, d]) for d in range(hd)) / math.sqrt(hd) for t in keys]
            m = max(sc)
            w = [math.exp(x - m) for x in sc]
            out[r_, h] = sum(wi * v[ck[i] + t, j] for wi, t in zip(w, keys)) / sum(w)
    return out


@pytest.mark.parametrize("causal", [True, False])
def test_varlen_prefill_brute_force(causal):
    q, k, v, cq, ck = varlen_setup()
    np.testing.assert_allclose(ref.varlen_prefill_attention(q, k, v, cq, ck, causal),
                               brute_varlen(q, k, v, cq, ck, causal), rtol=0, atol=1e-12)


def check_varlen_block_diagonal_mask(causal=True):
    """The whole packed batch as ONE attention whose mask is block-diagonal
    (a query sees only its own sequence's keys) and, when causal, lower
    triangular within a block from the bottom-right corner."""
    q, k, v, cq, ck = varlen_setup(seed=62)
    Tq, nh, hd = q.shape
    nkv = k.shape[1]
    seg_q = np.searchsorted(cq, np.arange(Tq), side="right") - 1
    seg_k = np.searchsorted(ck, np.arange(k.shape[0]), side="right") - 1
    rel_q = np.arange(Tq) - cq[seg_q] + (ck[seg_q + 1] - ck[seg_q]) - (cq[seg_q + 1] - cq[seg_q])
    rel_k = np.arange(k.shape[0]) - ck[seg_k]
    mask = seg_q[:, None] == seg_k[None, :]
    if causal:
        mask &= rel_k[None, :] <= rel_q[:, None]
    want = np.zeros((Tq, nh, hd))
    for h in range(nh):
        j = h // (nh // nkv)
        s = np.where(mask, q[:, h] @ k[:, j].T / np.sqrt(hd), -np.inf)
        has = mask.any(axis=1)
        e = np.exp(s - np.where(has, s.max(axis=1), 0.0)[:, None])
        want[has, h] = (e[has] / e[has].sum(axis=1, keepdims=True)) @ v[:, j]
    np.testing.assert_allclose(ref.varlen_prefill_attention(q, k, v, cq, ck, causal), want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_varlen_prefill_is_block_diagonal_attention(causal):
    check_varlen_block_diagonal_mask(causal)


def test_varlen_prefill_equals_padded_prefill():
    """Packing and padding give the same rows: the padded prefill over
    [B, nh, S_max, hd] queries with kv_lens and bottom-right positions."""
    q, k, v, cq, ck = varlen_setup(seed=63, q_lens=(3, 5, 1, 4), k_lens=(5, 5, 1, 9))
    B = len(cq) - 1
    nh, hd = q.shape[1], q.shape[2]
    nkv = k.shape[1]
    S, cap = int(np.diff(cq).max()), int(np.diff(ck).max())
    qp = np.zeros((B, nh, S, hd))
    kp, vp = np.zeros((B, nkv, cap, hd)), np.zeros((B, nkv, cap, hd))
    pos = np.zeros((B, S), dtype=np.int64)
    for b in range(B):
        Sq, Sk = cq[b + 1] - cq[b], ck[b + 1] - ck[b]
        qp[b, :, :Sq] = q[cq[b]:cq[b + 1]].transpose(1, 0, 2)
        kp[b, :, :Sk] = k[ck[b]:ck[b + 1]].transpose(1, 0, 2)
        vp[b, :, :Sk] = v[ck[b]:ck[b + 1]].transpose(1, 0, 2)
        pos[b] = Sk - Sq + np.arange(S)
    padded = ref.prefill_attention(qp, kp, vp, np.diff(ck), True, q_positions=pos)
    got = ref.varlen_prefill_attention(q, k, v, cq, ck, True)
    for b in range(B):
        np.testing.assert_allclose(got[cq[b]:cq[b + 1]], padded[b, :cq[b + 1] - cq[b]], rtol=0, atol=1e-12)


def test_varlen_prefill_special_cases():
    q, k, v, cq, ck = varlen_setup(seed=64)
    out = ref.varlen_prefill_attention(q, k, v, cq, ck, True)
    # a query of the 1-key sequence (index 3) sees exactly its one value
    nh, nkv = q.shape[1], k.shape[1]
    for h in range(nh):
        np.testing.assert_allclose(out[cq[3], h], v[ck[3], h // (nh // nkv)], rtol=0, atol=1e-15)
    # a sequence with no keys gives zero rows
    q2, k2, v2, cq2, ck2 = varlen_setup(seed=65, q_lens=(2, 3), k_lens=(0, 4))
    o2 = ref.varlen_prefill_attention(q2, k2, v2, cq2, ck2, False)
    assert np.all(o2[:2] == 0) and np.all(np.abs(o2[2:]) > 0)
    # one sequence is the plain causal prefill
    q3, k3, v3, cq3, ck3 = varlen_setup(seed=66, q_lens=(6,), k_lens=(6,))
    plain = ref.prefill_attention(q3.transpose(1, 0, 2)[None], k3.transpose(1, 0, 2)[None],
                                  v3.transpose(1, 0, 2)[None], np.array([6]), True)[0]
    np.testing.assert_allclose(ref.varlen_prefill_attention(q3, k3, v3, cq3, ck3, True), plain, rtol=0, atol=1e-12)


def test_planted_varlen_key_offset_is_caught(monkeypatch):
    """Reading a sequence's keys one row late (an off-by-one in the key
    offsets) fails the block-diagonal pin."""
    orig = ref.varlen_prefill_attention

    def shifted(q, k, v, cq, ck, causal):
        ck2 = np.minimum(np.asarray(ck) + np.r_[0, np.ones(len(ck) - 2, dtype=int), 0], ck[-1])
        return orig(q, k, v, cq, ck2, causal)
    monkeypatch.setattr(ref, "varlen_prefill_attention", shifted)
    assert _fails(check_varlen_block_diagonal_mask)


# --------------------------------------------------------------------------
# output projection (custom-op overhead gist: LlamaAttention ends with the
# output projection; the decoder layer adds the residual)
# --------------------------------------------------------------------------
def test_output_projection_brute_force():
    r = rng(71)
    T, nh, hd, D = 3, 4, 2, 5
    o, w, res = r.normal(size=(T, nh, hd)), r.normal(size=(D, nh * hd)), r.normal(size=(T, D))
    want = np.zeros((T, D))
    for t in range(T):
        for n in range(D):
            acc = float(res[t, n])
            for h in range(nh):
                for d in range(hd):
                    acc += float(o[t, h, d]) * float(w[n, h * hd + d])
            want[t, n] = acc
    np.testing.assert_allclose(ref.output_projection(o, w, res), want, rtol=0, atol=1e-12)


def check_output_projection_is_a_sum_over_heads():
    """The head-split form a fused epilogue computes: each head's output
    times its own hd-column slice of W_o, summed over heads."""
    r = rng(72)
    B, S, nh, hd, D = 2, 3, 4, 8, 16
    o, w = r.normal(size=(B, S, nh, hd)), r.normal(size=(D, nh * hd))
    want = sum(o[:, :, h] @ w[:, h * hd:(h + 1) * hd].T for h in range(nh))
    np.testing.assert_allclose(ref.output_projection(o, w), want, rtol=0, atol=1e-12)


def test_output_projection_is_a_sum_over_heads():
    check_output_projection_is_a_sum_over_heads()


def test_output_projection_zero_weight_passes_the_residual():
    """The gist initialises its projections to zero: the layer then returns
    the residual stream unchanged."""
    r = rng(73)
    res = r.normal(size=(2, 3, 12))
    np.testing.assert_array_equal(ref.output_projection(r.normal(size=(2, 3, 3, 4)), np.zeros((12, 12)), res), res)


def test_layer_prefill_then_decode_equals_one_prefill():
    """The whole attention layer (projection, RoPE, attention, output
    projection): a prompt's prefill followed by decode steps gives, token by
    token, the rows of one causal prefill over all the tokens."""
    r = rng(74)
    D, nh, nkv, hd, P, T = 16, 4, 2, 4, 5, 3
    x = r.normal(size=(1, P + T, D))
    w = r.normal(size=((nh + 2 * nkv) * hd, D)) * 0.3
    wo = r.normal(size=(D, nh * hd)) * 0.3
    cap = P + T
    z = np.zeros((1, nkv, cap, hd))
    pos_all = np.arange(P + T)[None]
    q, kc, vc = ref.qkv_rope_project(x, w, pos_all, nh, nkv, hd, 1e4, z, z)
    full = ref.output_projection(ref.prefill_attention(q, kc, vc, np.array([P + T]), True), wo, x)
    q, kc, vc = ref.qkv_rope_project(x[:, :P], w, pos_all[:, :P], nh, nkv, hd, 1e4, z, z)
    rows = [ref.output_projection(ref.prefill_attention(q, kc, vc, np.array([P]), True), wo, x[:, :P])]
    for t in range(P, P + T):
        q, kc, vc = ref.qkv_rope_project(x[:, t:t + 1], w, np.array([[t]]), nh, nkv, hd, 1e4, kc, vc)
        o = ref.decode_attention(q[:, :, 0], kc, vc, np.array([t + 1]))
        rows.append(ref.output_projection(o[:, None], wo, x[:, t:t + 1]))
    np.testing.assert_allclose(np.concatenate(rows, axis=1), full, rtol=0, atol=1e-12)


def test_planted_head_major_concat_is_caught(monkeypatch):
    """Concatenating as [hd, nh] (channel-major) instead of head order fails
    the head-split pin."""
    orig = ref.output_projection

    def channel_major(attn_out, w_o, residual=None):
        o = np.asarray(attn_out)
        return orig(np.swapaxes(o, -1, -2).reshape(o.shape), w_o, residual)
    monkeypatch.setattr(ref, "output_projection", channel_major)
    assert _fails(check_output_projection_is_a_sum_over_heads)


# --------------------------------------------------------------------------
# library routine as a special case: torch's scaled_dot_product_attention
# (float64, CPU) computes the same attention when every sequence is full
# (top-left and bottom-right causal alignment coincide) and, for decode,
# per sequence over its first kv_len keys
# --------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("nh,nkv", [(8, 2), (4, 4), (6, 1)])
def test_prefill_equals_library_sdpa(causal, nh, nkv):
    import torch
    import torch.nn.functional as F
    r = rng(80 + nh + nkv)
    B, S, hd = 2, 37, 16
    q, k, v = r.normal(size=(B, nh, S, hd)), r.normal(size=(B, nkv, S, hd)), r.normal(size=(B, nkv, S, hd))
    lib = F.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
                                         is_causal=causal, enable_gqa=True).numpy()
    np.testing.assert_allclose(ref.prefill_attention(q, k, v, np.array([S, S]), causal), lib.transpose(0, 2, 1, 3),
                               rtol=0, atol=1e-12)


def test_decode_equals_library_sdpa_per_sequence():
    import torch
    import torch.nn.functional as F
    r = rng(83)
    B, nh, nkv, cap, hd = 3, 8, 2, 20, 16
    lens = np.array([20, 1, 9])
    q, kc, vc = r.normal(size=(B, nh, hd)), r.normal(size=(B, nkv, cap, hd)), r.normal(size=(B, nkv, cap, hd))
    got = ref.decode_attention(q, kc, vc, lens)
    for b, L in enumerate(lens):
        lib = F.scaled_dot_product_attention(torch.from_numpy(q[b][:, None]), torch.from_numpy(kc[b, :, :L]),
                                             torch.from_numpy(vc[b, :, :L]), enable_gqa=True).numpy()[:, 0]
        np.testing.assert_allclose(got[b], lib, rtol=0, atol=1e-12)


def test_rope_matches_the_hf_llama_rotary_embedding():
    """The RoPE reading (rotate_half pairs, inv_freq = theta^(-2i/hd)) is HF
    Llama's: its rotary embedding and apply_rotary_pos_emb rotate q and k the
    same way.  The library forms its angles in float32, so the bound is its
    angle rounding (position x 2^-24 relative), far below the O(1) gap a
    different pairing, frequency or sign would leave."""
    import torch
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding, apply_rotary_pos_emb
    B, S, nh, nkv, hd = 2, 9, 4, 2, 64
    cfg = LlamaConfig(hidden_size=nh * hd, num_attention_heads=nh, num_key_value_heads=nkv, head_dim=hd,
                      rope_theta=10000.0, max_position_embeddings=4096)
    r = rng(84)
    q, k = r.normal(size=(B, nh, S, hd)), r.normal(size=(B, nkv, S, hd))
    pos = np.array([[0, 1, 2, 3, 17, 64, 99, 5, 40], [9, 8, 7, 6, 5, 4, 3, 2, 1]])
    cos, sin = LlamaRotaryEmbedding(cfg)(torch.from_numpy(q), torch.from_numpy(pos))
    qe, ke = apply_rotary_pos_emb(torch.from_numpy(q), torch.from_numpy(k), cos.double(), sin.double())
    for mine, lib in ((ref.apply_rope(q.transpose(0, 2, 1, 3), pos, 10000.0), qe),
                      (ref.apply_rope(k.transpose(0, 2, 1, 3), pos, 10000.0), ke)):
        np.testing.assert_allclose(mine.transpose(0, 2, 1, 3), lib.numpy(), rtol=0, atol=2e-4)


@pytest.mark.parametrize("nh,nkv", [(4, 2), (4, 4), (4, 1)])
def test_layer_equals_hf_llama_attention(nh, nkv):
    """The whole layer as the pages state it (fused projection sliced into
    q/k/v, RoPE on q and k, causal attention with the h -> h/g map, output
    projection) equals HF's LlamaAttention (eager, float64; its rotary
    angles are float32, hence the bound) with q/k/v_proj cut from W_qkv."""
    import torch
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaAttention, LlamaRotaryEmbedding
    B, S, D, hd = 2, 11, 64, 16
    cfg = LlamaConfig(hidden_size=D, num_attention_heads=nh, num_key_value_heads=nkv, head_dim=hd,
                      rope_theta=10000.0, attention_bias=False, max_position_embeddings=512)
    cfg._attn_implementation = "eager"
    att = LlamaAttention(cfg, layer_idx=0).double()
    r = rng(85 + nkv)
    x = r.normal(size=(B, S, D))
    w = r.normal(size=((nh + 2 * nkv) * hd, D)) * 0.3
    wo = r.normal(size=(D, nh * hd)) * 0.3
    q_end, k_end = nh * hd, (nh + nkv) * hd
    with torch.no_grad():
        att.q_proj.weight.copy_(torch.from_numpy(w[:q_end]))
        att.k_proj.weight.copy_(torch.from_numpy(w[q_end:k_end]))
        att.v_proj.weight.copy_(torch.from_numpy(w[k_end:]))
        att.o_proj.weight.copy_(torch.from_numpy(wo))
        pos = np.tile(np.arange(S), (B, 1))
        cos, sin = LlamaRotaryEmbedding(cfg)(torch.from_numpy(x), torch.from_numpy(pos))
        mask = torch.full((S, S), float("-inf"), dtype=torch.float64).triu(1)[None, None].expand(B, 1, S, S)
        lib, _ = att(torch.from_numpy(x), (cos.double(), sin.double()), mask)
    z = np.zeros((B, nkv, S, hd))
    q, kc, vc = ref.qkv_rope_project(x, w, pos, nh, nkv, hd, 10000.0, z, z)
    mine = ref.output_projection(ref.prefill_attention(q, kc, vc, np.full(B, S), True), wo)
    np.testing.assert_allclose(mine, lib.numpy(), rtol=0, atol=1e-6 * np.max(np.abs(mine)))
