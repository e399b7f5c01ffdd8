"""FP8 prefill with incoherent processing on the GPU (gqa_fp8_quantize_qkv +
gqa_attn_prefill_fp8) against the float64 FP8 oracle (oracle/fp8_ref.py):
the random-sign Hadamard rotation, per-tensor amax scales and e4m3 codes of
the quantiser, then the attention on the quantised tensors.

Codes are compared one by one: they must equal the oracle's rounding of the
rotated, scaled value, except where that value lies within float32 rounding
of a midpoint between two e4m3 values (the kernel decides in float32), where
either neighbour is accepted.  The attention output is compared with exact
softmax attention (float64) over the oracle's dequantised q, k and v, under
a bound derived from e4m3: the kernel rounds each probability to e4m3 (at
most 2^-4 relative) before P.V, so an output element may move by up to
2^-4 * sum_t w_t |v_tc| (w the exact softmax weights), plus half a bf16 ulp
for its own rounding and 2e-3 of the row scale for the rare code flips and
float32 accumulation."""
import numpy as np
import pytest
import torch

import mqa_attention_qkv_b200 as gqa
import workloads as W
from oracle import fp8_ref as f8
from oracle import gqa_ref as ref
from tests._helpers import dev, dev_i32, half_ulp_bf16, host

pytestmark = pytest.mark.gpu


def _signs(hd, seed):
    return np.where(np.random.default_rng([seed, 9]).integers(0, 2, hd) == 1, -1, 1).astype(np.int8)


def _decode(codes: torch.Tensor) -> np.ndarray:
    return codes.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.float64)


def _run(q, k, v, lens, signs, causal):
    B, nh, S, hd = q.shape
    nkv, cap = k.shape[1], k.shape[2]
    q8 = torch.zeros((B, nh, S, hd), dtype=torch.uint8, device="cuda")
    k8 = torch.full((B, nkv, cap, hd), 0x55, dtype=torch.uint8, device="cuda")
    v8t = torch.full((B, nkv, hd, cap), 0x55, dtype=torch.uint8, device="cuda")
    amax = torch.full((3,), -1.0, device="cuda")
    ln = dev_i32(lens)
    gqa.gqa_fp8_quantize_qkv(q, k, v, ln, q8, k8, v8t, amax, signs=signs)
    out = torch.full((B, S, nh, hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    gqa.gqa_attn_prefill_fp8(q8, k8, v8t, amax, ln, causal, out)
    torch.cuda.synchronize()
    return q8, k8, v8t, amax.cpu().numpy().astype(np.float64), out


def _valid_rows(x, lens):
    """The cache rows below each sequence's kv_len, [n, hd]."""
    return np.concatenate([x[b, :, :int(lens[b])].reshape(-1, x.shape[-1]) for b in range(x.shape[0])])


def _check_codes(got_vals, t, what):
    """got_vals: decoded GPU codes; t: the oracle's value before rounding."""
    want = f8.round_e4m3(t)
    bad = got_vals != want
    if np.any(bad):
        grid = f8.e4m3_values()
        tb, gb, wb = t[bad], got_vals[bad], want[bad]
        mid = (gb + wb) / 2.0
        near_mid = np.abs(tb - mid) <= 1e-5 * np.maximum(np.abs(tb), 2.0 ** -9)
        ig, iw = np.searchsorted(grid, gb), np.searchsorted(grid, wb)
        assert np.all(near_mid & (np.abs(ig - iw) == 1)), \
            f"{what}: {int((~(near_mid & (np.abs(ig - iw) == 1))).sum())} codes differ from the oracle's rounding"
    return int(bad.sum())


def _inputs(B, S, nh, nkv, hd, cap, seed, outliers):
    if outliers:
        q, k, v = W.outlier_qkv(B, S, nh, nkv, hd, seed)
        qf, kf, vf = q.f64, k.f64, v.f64
    else:
        qf = W.normal_tensor((B, nh, S, hd), seed, 0, "bf16").f64
        kf = W.normal_tensor((B, nkv, S, hd), seed, 1, "bf16").f64
        vf = W.normal_tensor((B, nkv, S, hd), seed, 2, "bf16").f64
    # caches of capacity cap: rows past S hold NaN, which must never be read
    kc = np.full((B, nkv, cap, hd), np.nan)
    vc = np.full((B, nkv, cap, hd), np.nan)
    kc[:, :, :S], vc[:, :, :S] = kf, vf
    return qf, kc, vc


def _to_dev(x):
    return torch.from_numpy(x.astype(np.float32)).cuda().to(torch.bfloat16)


def _oracle_quant(qf, kc, vc, lens, signs):
    """The oracle's rotation, amax and rounding (values before rounding too)."""
    hd = qf.shape[-1]
    M = f8.random_sign_hadamard(hd, signs) if signs is not None else np.eye(hd)
    qr, kr = qf @ M, kc @ M
    amax = [np.max(np.abs(qr)), np.max(np.abs(_valid_rows(kr, lens))), np.max(np.abs(_valid_rows(vc, lens)))]
    return (qr, kr, vc), amax


def _bound(q, k, v, lens, rows, causal):
    """Exact attention rows over the dequantised tensors and the per-element bound."""
    B, nh, S, hd = q.shape
    g = nh // k.shape[1]
    outs, lims = [], []
    for b, h, s in rows:
        L = int(lens[b])
        n_vis = min(L, L - S + s + 1) if causal else L
        o, w = ref.attend_row(q[b, h, s], k[b, h // g, :L], v[b, h // g, :L], n_vis)
        wv = w @ np.abs(v[b, h // g, :n_vis]) if n_vis > 0 else np.zeros(hd)
        outs.append(o)
        lims.append(2.0 ** -4 * wv)
    o = np.stack(outs)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True))
    return o, np.stack(lims) + half_ulp_bf16(o) + 2e-3 * np.minimum(1.0, rms)


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("nkv", [4, 1])
def test_fp8_quantize_and_prefill_parity(nkv, causal, rotate):
    B, S, nh, hd, cap = 2, 384, 8, 128, 448
    lens = np.array([S, S], dtype=np.int32)
    qf, kc, vc = _inputs(B, S, nh, nkv, hd, cap, 61 + nkv, outliers=True)
    signs = _signs(hd, 5) if rotate else None
    q8, k8, v8t, amax, out = _run(_to_dev(qf), _to_dev(kc), _to_dev(vc), lens, signs, causal)

    (qr, kr, vr), amax_r = _oracle_quant(qf, kc, vc, lens, signs)
    np.testing.assert_allclose(amax, amax_r, rtol=2e-6)
    sc = [a / 448.0 for a in amax]
    _check_codes(_decode(q8), qr / sc[0], "q codes")
    kg, vg = _decode(k8), _decode(v8t).transpose(0, 1, 3, 2)
    for b in range(B):
        L = int(lens[b])
        _check_codes(kg[b, :, :L], kr[b, :, :L] / sc[1], "k codes")
        _check_codes(vg[b, :, :L], vr[b, :, :L] / sc[2], "v codes")
        assert np.all(kg[b, :, L:] == 0) and np.all(vg[b, :, L:] == 0)

    # attention over the oracle's dequantised tensors (its own codes, its own scales)
    qq = f8.round_e4m3(qr / (amax_r[0] / 448.0)) * (amax_r[0] / 448.0)
    kq = f8.round_e4m3(np.nan_to_num(kr) / (amax_r[1] / 448.0)) * (amax_r[1] / 448.0)
    vq = f8.round_e4m3(np.nan_to_num(vr) / (amax_r[2] / 448.0)) * (amax_r[2] / 448.0)
    r = np.random.default_rng(3)
    rows = [(int(r.integers(B)), int(r.integers(nh)), int(r.integers(S))) for _ in range(48)]
    rows += [(0, 0, 0), (B - 1, nh - 1, S - 1), (0, 1, 127), (1, 2, 128), (0, 3, 255), (1, 4, 256)]
    want, lim = _bound(qq, kq, vq, lens, rows, causal)
    oh = host(out)
    got = np.stack([oh[b, s, h] for b, h, s in rows])
    assert np.all(np.isfinite(got))
    err = np.abs(got - want)
    assert np.all(err <= lim), f"fp8 prefill: worst err/bound {float(np.max(err / lim)):.3f}"


def test_fp8_rotation_reduces_error_on_outliers():
    """The page's claim, measured on the GPU path: with 0.1% of the channels
    x20, FP8 attention error against the exact (unquantised) attention is
    smaller with the random-sign Hadamard rotation than without."""
    B, S, nh, nkv, hd = 1, 512, 8, 8, 128
    lens = np.array([S], dtype=np.int32)
    qf, kc, vc = _inputs(B, S, nh, nkv, hd, S, 71, outliers=True)
    exact = ref.prefill_attention(qf, kc, vc, lens, False)             # [B, S, nh, hd]
    errs = {}
    for rot in (True, False):
        *_, out = _run(_to_dev(qf), _to_dev(kc), _to_dev(vc), lens, _signs(hd, 5) if rot else None, False)
        errs[rot] = float(np.sqrt(np.mean((host(out) - exact) ** 2)))
    assert errs[True] * 1.1 < errs[False], errs


def test_fp8_quantize_of_zero_tensors():
    B, S, nh, nkv, hd, cap = 1, 128, 2, 1, 128, 128
    z = torch.zeros((B, nh, S, hd), dtype=torch.bfloat16, device="cuda")
    zc = torch.zeros((B, nkv, cap, hd), dtype=torch.bfloat16, device="cuda")
    q8, k8, v8t, amax, out = _run(z, zc, zc, np.array([cap], dtype=np.int32), _signs(hd, 1), True)
    assert np.all(amax == 0)
    for codes in (q8, k8, v8t):     # +0 or -0 (the rotation of a zero row may carry a sign)
        assert np.all(_decode(codes) == 0.0)
    assert torch.all(out == 0)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("nkv", W.LONG_PREFILL.extra["n_kv_heads_cases"])
def test_fp8_long_prefill_outliers(nkv, causal):
    """The 2 x 8192 outlier workload (16 heads, hd 128) at full size, sampled rows."""
    wl = W.LONG_PREFILL
    B, S = wl.batch_seq[0]
    nh, hd = wl.shape.n_heads, wl.shape.head_dim
    q, k, v = W.outlier_qkv(B, S, nh, nkv, hd, wl.seed + nkv)
    lens = np.full(B, S, dtype=np.int32)
    signs = _signs(hd, wl.seed)
    q8, k8, v8t, amax, out = _run(dev(q), dev(k), dev(v), lens, signs, causal)
    (qr, kr, vr), amax_r = _oracle_quant(q.f64, k.f64, v.f64, lens, signs)
    np.testing.assert_allclose(amax, amax_r, rtol=2e-6)
    sc = [a / 448.0 for a in amax_r]
    qq = f8.round_e4m3(qr / sc[0]) * sc[0]
    kq = f8.round_e4m3(kr / sc[1]) * sc[1]
    vq = f8.round_e4m3(vr / sc[2]) * sc[2]
    r = np.random.default_rng(4)
    rows = [(int(r.integers(B)), h, int(r.integers(S))) for h in range(nh) for _ in range(3)]
    rows += [(0, 0, 0), (1, nh - 1, S - 1)]
    want, lim = _bound(qq, kq, vq, lens, rows, causal)
    oh = host(out)
    got = np.stack([oh[b, s, h] for b, h, s in rows])
    err = np.abs(got - want)
    assert np.all(err <= lim), f"fp8 long prefill: worst err/bound {float(np.max(err / lim)):.3f}"
