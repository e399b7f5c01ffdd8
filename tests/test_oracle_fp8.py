"""Pins for the FP8 / incoherent-processing oracle (CPU only).

They tie oracle/fp8_ref.py to what the FlashAttention-3 summary (section "FP8
低精度とincoherent processing") and the mathematics fix: the Hadamard matrix
and its orthogonality, the invariance of the scores under one rotation of Q
and K, the e4m3 code table decoded bit by bit, round-to-nearest-even against
a literal search, and the page's claim that the rotation reduces the FP8
error on inputs with outliers.  A planted mistake (rotating Q only) fails.
"""
import numpy as np
import pytest

from oracle import fp8_ref as f8


def test_sylvester_hadamard_small_orders_and_orthogonality():
    np.testing.assert_array_equal(f8.sylvester_hadamard(2), [[1, 1], [1, -1]])
    np.testing.assert_array_equal(f8.sylvester_hadamard(4),
                                  [[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]])
    for d in (8, 32, 64, 128):
        h = f8.sylvester_hadamard(d)
        assert set(np.unique(h)) == {-1.0, 1.0}
        np.testing.assert_array_equal(h @ h.T, d * np.eye(d))


@pytest.mark.parametrize("d", [32, 64, 128])
def test_random_sign_hadamard_is_orthogonal(d):
    signs = np.where(np.random.default_rng(d).random(d) < 0.5, -1.0, 1.0)
    m = f8.random_sign_hadamard(d, signs)
    np.testing.assert_allclose(m @ m.T, np.eye(d), rtol=0, atol=1e-12)
    np.testing.assert_allclose(m.T @ m, np.eye(d), rtol=0, atol=1e-12)


def check_rotation_leaves_scores_and_attention_unchanged(rotate_k=True):
    r = np.random.default_rng(7)
    d = 64
    q, k, v = r.standard_normal((2, 9, d)), r.standard_normal((2, 11, d)), r.standard_normal((2, 11, d))
    m = f8.random_sign_hadamard(d, np.where(r.random(d) < 0.5, -1.0, 1.0))
    k2 = k @ m if rotate_k else k
    np.testing.assert_allclose((q @ m) @ np.swapaxes(k2, -1, -2), q @ np.swapaxes(k, -1, -2), rtol=0, atol=1e-12)
    np.testing.assert_allclose(f8.attention(q @ m, k2, v), f8.attention(q, k, v), rtol=0, atol=1e-12)


def test_rotation_leaves_scores_and_attention_unchanged():
    check_rotation_leaves_scores_and_attention_unchanged()


def test_planted_rotation_of_q_only_is_caught():
    with pytest.raises(AssertionError):
        check_rotation_leaves_scores_and_attention_unchanged(rotate_k=False)


def decode_e4m3(code):
    """Literal bit decoding of one e4m3 code, written out again here."""
    s = -1.0 if code >> 7 else 1.0
    e, m = (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return None
    return s * (m * 2.0 ** -9 if e == 0 else (8 + m) * 2.0 ** (e - 10))


def test_e4m3_code_table():
    vals = f8.e4m3_values()
    decoded = sorted({decode_e4m3(c) for c in range(256) if decode_e4m3(c) is not None})
    np.testing.assert_array_equal(vals, decoded)
    assert len(vals) == 253                       # 254 finite codes, +0 and -0 equal
    assert vals.max() == 448.0 and vals.min() == -448.0
    pos = vals[vals > 0]
    assert pos[0] == 2.0 ** -9 and 2.0 ** -6 in pos and 1.0 in pos
    one = np.searchsorted(vals, 1.0)
    assert vals[one + 1] - vals[one] == 0.125     # 3 mantissa bits: step 1/8 in [1, 2)


def brute_round(x):
    """Nearest finite e4m3 value by exhaustive search over the codes, ties to
    the even code, saturating."""
    best = None
    for c in range(256):
        v = decode_e4m3(c)
        if v is None:
            continue
        key = (abs(min(max(x, -448.0), 448.0) - v), c & 1)
        if best is None or key < best[0]:
            best = (key, v)
    return best[1]


def test_round_e4m3_against_exhaustive_search():
    r = np.random.default_rng(8)
    xs = np.concatenate([r.standard_normal(300) * 10.0, r.standard_normal(100) * 1e-3, [0.0, 1000.0, -1000.0],
                         [1.0 + 1 / 16, 1.0 + 3 / 16, -(1.0 + 1 / 16), 2.0 ** -10, 3 * 2.0 ** -10]])
    got = f8.round_e4m3(xs)
    want = np.array([brute_round(float(x)) for x in xs])
    np.testing.assert_array_equal(np.abs(got), np.abs(want))
    np.testing.assert_array_equal(got[got != 0], want[got != 0])
    # ties to even: 1 + 1/16 lies between 1 (code 0x38) and 1.125 (0x39)
    assert f8.round_e4m3(np.array([1.0 + 1 / 16]))[0] == 1.0
    assert f8.round_e4m3(np.array([1.0 + 3 / 16]))[0] == 1.25
    vals = f8.e4m3_values()
    np.testing.assert_array_equal(f8.round_e4m3(vals), vals)      # the grid is fixed


def test_quantize_maps_amax_to_the_largest_code():
    t = np.random.default_rng(9).standard_normal((5, 7)) * 3.0
    dq, scale = f8.quantize_e4m3(t)
    i = np.unravel_index(np.argmax(np.abs(t)), t.shape)
    assert scale == pytest.approx(np.max(np.abs(t)) / 448.0, rel=1e-15)
    assert dq[i] == pytest.approx(t[i], rel=1e-15)
    assert np.max(np.abs(dq - t) / np.maximum(np.abs(t), 2 ** -6 * scale)) <= 2 ** -4 + 1e-12


def test_incoherent_processing_reduces_fp8_error_with_outliers():
    """The page's experiment shape: N(0,1) Q, K, V with 0.1% of the entries
    made large (x20 here, the outlier factor of the long-prefill workload).
    The rotation lowers the error of FP8 attention against exact attention.
    The page reports 2.6x for a setup it does not state; with per-tensor
    e4m3 scales (the reading taken) the reduction is about 1.4x, so this pins
    the direction with a margin: at least 1.25x."""
    d = 128
    q, k, v = f8.outlier_inputs((4, 256, d), 0.001, 20.0, seed=10)
    exact = f8.attention(q, k, v)
    m = f8.random_sign_hadamard(d, np.where(np.random.default_rng(11).random(d) < 0.5, -1.0, 1.0))
    err_plain = np.sqrt(np.mean((f8.fp8_attention(q, k, v) - exact) ** 2))
    err_rot = np.sqrt(np.mean((f8.fp8_attention(q, k, v, rotation=m) - exact) ** 2))
    assert err_rot * 1.25 <= err_plain, (err_plain, err_rot)


def test_round_e4m3_matches_torch_float8_cast_in_range():
    """Inside the finite range the rounding is the library's e4m3 cast
    (torch.float8_e4m3fn: nearest, ties to even), checked on random values
    and on every exact midpoint between neighbouring codes."""
    import torch
    grid = f8.e4m3_values()
    r = np.random.default_rng(12)
    x = np.concatenate([r.standard_normal(20000) * 50.0, r.standard_normal(5000) * 1e-2, grid,
                        (grid[1:] + grid[:-1]) / 2.0]).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(f8.round_e4m3(x.astype(np.float64)), lib)
