"""GPU parity: the CUDA library (called through its C ABI) against the float64
oracle on the same seeded inputs.  Small cases are compared element by
element; the five workloads run at their full sizes and are compared on
sampled rows that the oracle computes one by one."""
import numpy as np
import pytest
import torch

import mqa_attention_qkv_b200 as gqa
import workloads as W
from oracle import gqa_ref as ref
from tests._helpers import bits, dev, dev_i32, gate, host

pytestmark = pytest.mark.gpu

TORCH_DT = {"bf16": torch.bfloat16, "f32": torch.float32}
SENTINEL = {"bf16": np.uint16(0x7FA5), "f32": np.uint32(0x7FC0_1234)}  # NaN payloads


def sentinel_cache(shape, dtype):
    if dtype == "bf16":
        return W.Tensor(np.full(shape, SENTINEL["bf16"], dtype=np.uint16), "bf16")
    return W.Tensor(np.full(shape, SENTINEL["f32"], dtype=np.uint32).view(np.float32), "f32")


def nan_padded(B, nkv, cap, hd, lens, seed, tid, dtype):
    return W.decode_cache(seed, tid, B, nkv, cap, hd, lens, dtype=dtype)


def run_project(x, w, pos, nh, nkv, hd, cap, dtype, theta=10000.0, kc=None, vc=None):
    B, S, _ = x.shape
    xd, wd = dev(x), dev(w)
    q = torch.empty((B, nh, S, hd), dtype=TORCH_DT[dtype], device="cuda")
    kc = kc if kc is not None else dev(sentinel_cache((B, nkv, cap, hd), dtype))
    vc = vc if vc is not None else dev(sentinel_cache((B, nkv, cap, hd), dtype))
    gqa.qkv_rope_project(xd, wd, dev_i32(pos), nh, nkv, hd, theta, q, kc, vc)
    return q, kc, vc


# --------------------------------------------------------------------------
# a1-a3: projection + RoPE + scatter
# --------------------------------------------------------------------------
QKV_CASES = [
    # dtype, B, S, hidden, nh, nkv, hd, cap, scattered positions
    ("f32", 1, 128, 256, 8, 2, 32, 128, False),
    ("f32", 2, 19, 96, 4, 4, 64, 40, True),
    ("bf16", 2, 37, 192, 4, 2, 64, 64, True),
    ("bf16", 3, 130, 256, 8, 1, 128, 200, True),
    ("bf16", 1, 5, 64, 2, 1, 32, 8, False),
    ("bf16", 2, 200, 2048, 32, 4, 64, 256, False),
    ("bf16", 1, 333, 520, 6, 2, 128, 400, True),
    ("bf16", 3, 150, 136, 3, 1, 64, 160, True),     # N = 320 (partial 256-tile), K tail, T = 450
    ("bf16", 2, 300, 256, 12, 2, 32, 320, False),   # hd 32: 8 heads per tile
    ("bf16", 2, 1024, 512, 16, 4, 64, 1024, True),  # 96 tiles: several per persistent CTA
    ("bf16", 2, 2000, 512, 16, 4, 64, 2048, True),  # 192 tiles, T tail: the last wave's 44 tiles as 88 halves
    ("bf16", 1, 4000, 256, 8, 2, 128, 4096, False),  # the same split at hd 128 (a half tile is one head)
    ("bf16", 3, 2000, 256, 10, 2, 64, 2048, True),  # N = 896: the last column tile's second half lies past N
    ("bf16", 2, 70, 100, 4, 2, 64, 80, True),       # hidden % 8 != 0: the SIMT path
    # 128 tokens or fewer over tiles that fill less than half of the SMs: the K
    # split across a cluster (ranks' partial sums added by the leader)
    ("bf16", 1, 128, 2048, 32, 4, 64, 128, False),  # TinyLlama 1 x 128: 40 tiles x 2 ranks
    ("bf16", 1, 100, 2048, 32, 4, 64, 160, True),   # ragged T: rows past T masked in every rank
    ("bf16", 1, 96, 4096, 32, 8, 128, 96, True),    # hd 128: 48 tiles of 128 columns x 2 ranks
    ("bf16", 2, 50, 1024, 16, 4, 32, 64, True),     # hd 32: 12 tiles x 2 ranks
    # few tokens, hidden % 64 == 0 and the hidden states fit in shared memory:
    # the TMA-ring kernel, every token-count variant
    ("bf16", 3, 1, 2048, 32, 4, 64, 16, True),
    ("bf16", 8, 1, 6144, 48, 1, 128, 40, True),     # 400 units: several per CTA, 12 stages each
    ("bf16", 5, 1, 4096, 16, 4, 64, 8, True),
    ("bf16", 8, 1, 7168, 8, 1, 128, 8, True),       # 112 column blocks, 14 stages
    ("bf16", 4, 4, 1088, 8, 2, 64, 32, True),       # T = 16: 17 column blocks
    ("bf16", 3, 4, 3584, 4, 2, 128, 16, True),      # T = 12
    ("bf16", 3, 9, 768, 6, 3, 128, 64, False),
    ("bf16", 8, 5, 256, 12, 2, 32, 9, True),
    # few tokens, hidden % 64 != 0: the register-streaming kernel, every token-count variant
    ("bf16", 5, 1, 520, 8, 2, 64, 8, True),
    ("bf16", 4, 3, 520, 8, 2, 128, 8, True),
    ("bf16", 2, 10, 1000, 6, 1, 128, 16, True),
    ("bf16", 1, 64, 136, 4, 4, 64, 64, False),
]


@pytest.mark.parametrize("case", QKV_CASES, ids=lambda c: "-".join(map(str, c)))
def test_qkv_rope_project_parity(case):
    dtype, B, S, hidden, nh, nkv, hd, cap, scatter = case
    shape = W.LayerShape(hidden, nh, nkv, hd)
    x, w, pos = W.layer_inputs(shape, B, S, seed=11, dtype=dtype)
    if scatter:
        r = np.random.default_rng(5)
        pos = np.stack([r.permutation(cap)[:S] for _ in range(B)]).astype(np.int32)
    q, kc, vc = run_project(x, w, pos, nh, nkv, hd, cap, dtype)
    sent = sentinel_cache((B, nkv, cap, hd), dtype)
    q_ref, kc_ref, vc_ref = ref.qkv_rope_project(x.f64, w.f64, pos, nh, nkv, hd, 10000.0,
                                                 np.zeros((B, nkv, cap, hd)), np.zeros((B, nkv, cap, hd)))
    gate(host(q), q_ref, dtype, "q_out")
    written = np.zeros((B, cap), dtype=bool)
    for b in range(B):
        written[b, pos[b]] = True
    kh, vh = host(kc), host(vc)
    for b in range(B):
        gate(kh[b][:, written[b]], kc_ref[b][:, written[b]], dtype, "k_cache")
        gate(vh[b][:, written[b]], vc_ref[b][:, written[b]], dtype, "v_cache")
    # untouched slots keep their exact bits
    kb, vb = bits(kc), bits(vc)
    sb = sent.store.view(np.uint16 if dtype == "bf16" else np.uint32)
    for b in range(B):
        assert np.array_equal(kb[b][:, ~written[b]], sb[b][:, ~written[b]])
        assert np.array_equal(vb[b][:, ~written[b]], sb[b][:, ~written[b]])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hd", [32, 64, 128])
def test_kv_cache_layout_bit_exact(dtype, hd):
    """One-hot hidden states and small-integer weights make every projected
    value an exact integer: V rows land bit-exactly at slot = position, K and Q
    too for tokens at position 0 (rotation by zero)."""
    B, S, D, nh, nkv, cap = 2, 9, 64, 4, 2, 24
    N = (nh + 2 * nkv) * hd
    w_int = ((np.arange(N * D).reshape(N, D) * 7919) % 61 - 30).astype(np.float32)
    x_int = np.zeros((B, S, D), dtype=np.float32)
    for b in range(B):
        for s in range(S):
            x_int[b, s, (3 * b + 5 * s) % D] = 1.0
    x = W.Tensor(W.bf16_bits(x_int), "bf16") if dtype == "bf16" else W.Tensor(x_int, "f32")
    w = W.Tensor(W.bf16_bits(w_int), "bf16") if dtype == "bf16" else W.Tensor(w_int, "f32")
    pos = np.array([[0, 5, 9, 11, 13, 17, 19, 21, 23], [23, 0, 2, 4, 6, 8, 10, 12, 14]], dtype=np.int32)
    q, kc, vc = run_project(x, w, pos, nh, nkv, hd, cap, dtype)
    kh, vh, qh = host(kc), host(vc), host(q)
    for b in range(B):
        for s in range(S):
            col = (3 * b + 5 * s) % D
            p = pos[b, s]
            v_want = w_int[(nh + nkv) * hd:, col].reshape(nkv, hd)
            assert np.array_equal(vh[b, :, p], v_want), (b, s)
            if p == 0:
                assert np.array_equal(kh[b, :, p], w_int[nh * hd:(nh + nkv) * hd, col].reshape(nkv, hd))
                assert np.array_equal(qh[b, :, s], w_int[:nh * hd, col].reshape(nh, hd))
    # unwritten slots keep the sentinel bits
    kb = bits(kc)
    sent = SENTINEL[dtype]
    for b in range(B):
        free = sorted(set(range(cap)) - set(pos[b].tolist()))
        assert np.all(kb[b][:, free] == sent)


def test_out_of_range_position_sets_error_and_skips_row():
    dtype, B, S, hidden, nh, nkv, hd, cap = "bf16", 1, 4, 64, 2, 1, 64, 8
    x, w, _ = W.layer_inputs(W.LayerShape(hidden, nh, nkv, hd), B, S, seed=3, dtype=dtype)
    pos = np.array([[0, 3, 8, -1]], dtype=np.int32)
    gqa.gqa_device_error()  # clear
    q, kc, vc = run_project(x, w, pos, nh, nkv, hd, cap, dtype)
    assert gqa.gqa_device_error() & 1
    kb = bits(kc)
    assert np.all(kb[0, :, [1, 2, 4, 5, 6, 7]] == SENTINEL["bf16"])
    assert np.all(np.isfinite(host(q)))


# --------------------------------------------------------------------------
# a4: prefill attention
# --------------------------------------------------------------------------
def attn_inputs(B, nh, nkv, S, hd, cap, lens, dtype, seed):
    q = W.normal_tensor((B, nh, S, hd), seed, 0, dtype)
    kc = nan_padded(B, nkv, cap, hd, lens, seed, 1, dtype)
    vc = nan_padded(B, nkv, cap, hd, lens, seed, 2, dtype)
    return q, kc, vc


PREFILL_CASES = []
for _hd in (32, 64, 128):
    for _g, _nkv in ((1, 2), (2, 2), (4, 2), (8, 1), (32, 1)):
        for _S in (1, 7, 64, 129):
            PREFILL_CASES.append(("bf16", _hd, _g * _nkv, _nkv, _S))
PREFILL_CASES += [("f32", 32, 8, 2, 128), ("f32", 64, 4, 4, 37), ("f32", 128, 4, 1, 65)]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: "-".join(map(str, c)))
def test_prefill_parity(case, causal):
    dtype, hd, nh, nkv, S = case
    B = 2
    lens = np.array([S + 3, S], dtype=np.int32)        # ragged; first has a 3-key prefix
    cap = S + 11
    q, kc, vc = attn_inputs(B, nh, nkv, S, hd, cap, lens, dtype, seed=S + hd)
    out = torch.empty((B, S, nh, hd), dtype=TORCH_DT[dtype], device="cuda")
    gqa.gqa_attn_prefill(dev(q), dev(kc), dev(vc), dev_i32(lens), causal, out)
    want = ref.prefill_attention(q.f64, np.nan_to_num(kc.f64), np.nan_to_num(vc.f64), lens, causal)
    gate(host(out), want, dtype, f"prefill {case} causal={causal}")


def test_prefill_explicit_positions_and_empty_rows():
    dtype, B, nh, nkv, S, hd, cap = "bf16", 2, 4, 2, 6, 64, 16
    lens = np.array([10, 6], dtype=np.int32)
    q, kc, vc = attn_inputs(B, nh, nkv, S, hd, cap, lens, dtype, seed=99)
    qpos = np.array([[-1, 0, 2, 4, 9, 12], [5, 4, 3, 2, 1, 0]], dtype=np.int32)  # -1: no key; 12 > len
    out = torch.empty((B, S, nh, hd), dtype=torch.bfloat16, device="cuda")
    gqa.gqa_attn_prefill(dev(q), dev(kc), dev(vc), dev_i32(lens), True, out, q_positions=dev_i32(qpos))
    want = ref.prefill_attention(q.f64, np.nan_to_num(kc.f64), np.nan_to_num(vc.f64), lens, True, q_positions=qpos)
    got = host(out)
    assert np.all(got[0, 0] == 0.0)
    gate(got[:, 1:], want[:, 1:], dtype, "explicit positions")


# --------------------------------------------------------------------------
# packed variable-length prefill
# --------------------------------------------------------------------------
VARLEN_Q = [1, 127, 128, 129, 300, 0, 64, 257, 10]
VARLEN_K = [1, 127, 133, 129, 400, 3, 64, 257, 4]     # cached prefixes; the last has fewer keys than queries


def varlen_inputs(nh, nkv, hd, q_lens, k_lens, seed):
    cq = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(k_lens)]).astype(np.int32)
    q = W.normal_tensor((int(cq[-1]), nh, hd), seed, 0, "bf16")
    k = W.normal_tensor((int(ck[-1]), nkv, hd), seed, 1, "bf16")
    v = W.normal_tensor((int(ck[-1]), nkv, hd), seed, 2, "bf16")
    return q, k, v, cq, ck


def run_varlen(q, k, v, cq, ck, causal, max_q=None, out=None):
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    max_q = int(np.diff(cq).max()) if max_q is None else max_q
    gqa.gqa_attn_prefill_varlen(dev(q), dev(k), dev(v), dev_i32(cq), dev_i32(ck), max_q, causal, out)
    return out


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("hd,g,nkv", [(64, 1, 2), (64, 8, 1), (128, 4, 2), (128, 1, 1)])
def test_varlen_prefill_parity(hd, g, nkv, causal):
    """Packed sequences of ragged lengths (tile edges, an empty one, cached
    prefixes, fewer keys than queries) against the oracle's packed prefill."""
    nh = g * nkv
    q, k, v, cq, ck = varlen_inputs(nh, nkv, hd, VARLEN_Q, VARLEN_K, 80 + hd + g)
    gqa.gqa_device_error()
    got = host(run_varlen(q, k, v, cq, ck, causal))
    assert gqa.gqa_device_error() == 0
    want = ref.varlen_prefill_attention(q.f64, k.f64, v.f64, cq, ck, causal)
    if causal:   # the last sequence's first 6 queries see no key
        assert np.all(got[cq[-2]:cq[-2] + 6] == 0)
    gate(got.reshape(-1, hd), want.reshape(-1, hd), "bf16", f"varlen prefill hd{hd} g{g} causal={causal}")


@pytest.mark.parametrize("hd", [64, 128])
def test_varlen_prefill_matches_padded_bit_for_bit(hd):
    """The same sequences padded into [B, nh, S, hd] queries and a
    [B, nkv, cap, hd] cache, with the packed call's positions passed
    explicitly, give the same bits: only the tiles' addresses differ."""
    nh, nkv = 8, 2
    q_lens, k_lens = VARLEN_Q[:-1], VARLEN_K[:-1]
    q, k, v, cq, ck = varlen_inputs(nh, nkv, hd, q_lens, k_lens, 90 + hd)
    B, S, cap = len(q_lens), max(q_lens), max(k_lens)
    qp = np.zeros((B, nh, S, hd), dtype=np.uint16)
    kp = np.full((B, nkv, cap, hd), SENTINEL["bf16"], dtype=np.uint16)
    vp = np.full((B, nkv, cap, hd), SENTINEL["bf16"], dtype=np.uint16)
    pos = np.full((B, S), -1, dtype=np.int32)
    for b in range(B):
        qp[b, :, :q_lens[b]] = q.store[cq[b]:cq[b + 1]].transpose(1, 0, 2)
        kp[b, :, :k_lens[b]] = k.store[ck[b]:ck[b + 1]].transpose(1, 0, 2)
        vp[b, :, :k_lens[b]] = v.store[ck[b]:ck[b + 1]].transpose(1, 0, 2)
        pos[b, :q_lens[b]] = k_lens[b] - q_lens[b] + np.arange(q_lens[b])
    out_p = torch.empty((B, S, nh, hd), dtype=torch.bfloat16, device="cuda")
    gqa.gqa_attn_prefill(dev(W.Tensor(qp, "bf16")), dev(W.Tensor(kp, "bf16")), dev(W.Tensor(vp, "bf16")),
                         dev_i32(np.array(k_lens, dtype=np.int32)), True, out_p, q_positions=dev_i32(pos))
    packed = bits(run_varlen(q, k, v, cq, ck, True))
    padded = bits(out_p)
    for b in range(B):
        np.testing.assert_array_equal(packed[cq[b]:cq[b + 1]], padded[b, :q_lens[b]])


def test_varlen_prefill_bad_offsets_are_clamped_and_flagged():
    """Offsets past the packed tensors are clamped (nothing is written past
    the output) and flagged; so is a query run longer than max_seqlen_q."""
    nh, nkv, hd = 4, 1, 64
    q, k, v, cq, ck = varlen_inputs(nh, nkv, hd, [100, 200], [100, 200], 95)
    tq = int(cq[-1])
    big = torch.full((tq + 64, nh, hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    bad_q = cq.copy()
    bad_q[-1] = tq + 50
    bad_k = ck.copy()
    bad_k[-1] = int(ck[-1]) + 77
    gqa.gqa_device_error()
    run_varlen(q, k, v, bad_q, bad_k, True, max_q=256, out=big[:tq])
    assert gqa.gqa_device_error() & 16
    assert torch.isnan(big[tq:]).all()
    want = ref.varlen_prefill_attention(q.f64, k.f64, v.f64, cq, ck, True)
    gate(host(big[:tq]).reshape(-1, hd), want.reshape(-1, hd), "bf16", "clamped offsets")
    # max_seqlen_q shorter than a run: flagged; the rows the grid covers are right
    out = run_varlen(q, k, v, cq, ck, True, max_q=128)
    assert gqa.gqa_device_error() & 16
    got = host(out)
    gate(got[:100].reshape(-1, hd), want[:100].reshape(-1, hd), "bf16", "short max_seqlen_q")


# --------------------------------------------------------------------------
# a5-a6: decode
# --------------------------------------------------------------------------
def run_decode(q, kc, vc, lens, nh, dtype, kv_split=0):
    B, _, hd = q.shape
    nkv, cap = kc.shape[1], kc.shape[2]
    ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap, kv_split) // 4 + 1,
                     dtype=torch.float32, device="cuda")
    out = torch.empty((B, nh, hd), dtype=TORCH_DT[dtype], device="cuda")
    gqa.gqa_attn_decode(dev(q), dev(kc), dev(vc), dev_i32(lens), out, ws, kv_split=kv_split)
    return out


DECODE_CASES = [(dt, hd, g, nkv) for dt in ("bf16",) for hd in (32, 64, 128)
                for g, nkv in ((1, 4), (2, 2), (4, 2), (8, 1), (32, 1))]
DECODE_CASES += [("f32", 32, 4, 2), ("f32", 128, 1, 2), ("f32", 64, 8, 1)]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: "-".join(map(str, c)))
def test_decode_parity(case):
    dtype, hd, g, nkv = case
    nh = g * nkv
    lens = np.array([1, 63, 64, 65, 300, 1000, 7, 513], dtype=np.int32)
    B, cap = len(lens), 1024
    q = W.normal_tensor((B, nh, hd), 7, 0, dtype)
    kc = nan_padded(B, nkv, cap, hd, lens, 7, 1, dtype)
    vc = nan_padded(B, nkv, cap, hd, lens, 7, 2, dtype)
    want = ref.decode_attention(q.f64, np.nan_to_num(kc.f64), np.nan_to_num(vc.f64), lens)
    for split in (0, 64, 192):
        out = run_decode(q, kc, vc, lens, nh, dtype, kv_split=split)
        gate(host(out), want, dtype, f"decode {case} split={split}")


def test_decode_workspace_reuse_leaves_counters_zero():
    """One zero-filled workspace serves calls of different shapes in a row; the
    merge counters at its front are back at zero after each call."""
    ws = torch.zeros(8 << 20, dtype=torch.uint8, device="cuda")
    for seed, (B, nh, nkv, hd, cap, lens) in enumerate([
            (3, 32, 4, 128, 900, [900, 70, 511]),
            (5, 48, 1, 128, 700, [1, 700, 64, 65, 333]),
            (2, 8, 8, 64, 300, [300, 129])]):
        lens = np.array(lens, dtype=np.int32)
        q = W.normal_tensor((B, nh, hd), 40 + seed, 0, "bf16")
        kc = nan_padded(B, nkv, cap, hd, lens, 40 + seed, 1, "bf16")
        vc = nan_padded(B, nkv, cap, hd, lens, 40 + seed, 2, "bf16")
        out = torch.empty((B, nh, hd), dtype=torch.bfloat16, device="cuda")
        gqa.gqa_attn_decode(dev(q), dev(kc), dev(vc), dev_i32(lens), out, ws, kv_split=64)
        want = ref.decode_attention(q.f64, kc.f64, vc.f64, lens)
        gate(host(out), want, "bf16", f"reused workspace, case {seed}")
        n_counters = B * nkv * ((nh // nkv + 15) // 16)
        assert int(ws[:4 * n_counters].view(torch.int32).abs().sum()) == 0


def test_decode_split_count_invariance():
    """Workspace splits of 448, 256 and 64 keys (1, 2 and 7 splits) and the
    automatic cluster-merged split (7 CTAs of one tile each) agree to the
    float32 rounding of the merge."""
    dtype, hd, nh, nkv = "bf16", 128, 8, 1
    lens = np.array([448, 448], dtype=np.int32)
    B, cap = 2, 448
    q = W.normal_tensor((B, nh, hd), 8, 0, dtype)
    kc = nan_padded(B, nkv, cap, hd, lens, 8, 1, dtype)
    vc = nan_padded(B, nkv, cap, hd, lens, 8, 2, dtype)
    outs = [host(run_decode(q, kc, vc, lens, nh, dtype, kv_split=s)) for s in (448, 256, 64, 0)]
    for o in outs[1:]:
        assert np.max(np.abs(o - outs[0])) <= 2 ** -7 * np.max(np.abs(outs[0]))


@pytest.mark.parametrize("hd", (64, 128))
def test_decode_cluster_merge_ragged(hd):
    """Automatic split of a small ragged batch: each sequence's tiles are dealt
    out over a cluster of up to 8 CTAs, some of which get none (lengths 0, 1,
    64, 65), and the partials meet in distributed shared memory."""
    dtype, nh, nkv, cap = "bf16", 48, 1, 1040
    lens = np.array([0, 1, 64, 65, 528, 1040, 17, 900], dtype=np.int32)
    B = len(lens)
    q = W.normal_tensor((B, nh, hd), 12, 0, dtype)
    kc = nan_padded(B, nkv, cap, hd, lens, 12, 1, dtype)
    vc = nan_padded(B, nkv, cap, hd, lens, 12, 2, dtype)
    got = host(run_decode(q, kc, vc, lens, nh, dtype))
    assert np.all(got[0] == 0)
    want = ref.decode_attention(q.f64, np.nan_to_num(kc.f64), np.nan_to_num(vc.f64), lens)
    gate(got[1:], want[1:], dtype, "cluster-merged decode")


@pytest.mark.parametrize("hd,nh,nkv,B", [(64, 48, 1, 32), (128, 160, 1, 32), (128, 64, 2, 16)],
                         ids=["hd64-g48", "hd128-g160-two-head-groups", "hd128-g32-nkv2"])
def test_decode_tcgen05_large_batch(hd, nh, nkv, B):
    """Large batches with g > 16 (at least 2^18 cached key rows) take the
    tcgen05 decode: heads as the 128 MMA rows, each sequence's 64-key tiles
    dealt out over a cluster whose CTAs merge through distributed shared
    memory.  Ragged lengths with 0, 1 and tile edges; g = 160 has a second,
    partial head group."""
    dtype, cap = "bf16", 8192
    edge = [0, 1, 63, 64, 65, 1023, 1024, 1025, 2100, 4096, 8191, 8192]
    rng = np.random.default_rng(21)
    lens = np.array(edge + list(rng.integers(1, cap + 1, size=B - len(edge))), dtype=np.int32)[:B]
    q = W.normal_tensor((B, nh, hd), 14, 0, dtype)
    kc = nan_padded(B, nkv, cap, hd, lens, 14, 1, dtype)
    vc = nan_padded(B, nkv, cap, hd, lens, 14, 2, dtype)
    got = host(run_decode(q, kc, vc, lens, nh, dtype))
    assert np.all(got[0] == 0)
    want = ref.decode_attention(q.f64, np.nan_to_num(kc.f64), np.nan_to_num(vc.f64), lens)
    gate(got[1:], want[1:], dtype, "tcgen05 decode")


def _hn_lens(B, cap, seed, edge):
    rng = np.random.default_rng(seed)
    return np.array(edge + list(rng.integers(1, cap + 1, size=B - len(edge))), dtype=np.int32)[:B]


@pytest.mark.parametrize("g,nkv", [(32, 1), (24, 2), (48, 1), (64, 1)], ids=["g32", "g24-nkv2", "g48", "g64"])
def test_decode_keys_as_rows(g, nkv):
    """Large batches with 16 < g <= 64 at head_dim 128 whose cache is longer
    than the cluster kernel takes (here 20000 keys) use the decode with the
    keys as the 128 MMA rows and the heads as N (padded to a multiple of 16):
    equal tile ranges per SM, pieces merged through the workspace by the last
    piece of each (sequence, KV head).  Ragged lengths with 0, 1 and 128-key
    tile edges; two calls on one workspace leave its counters at zero."""
    dtype, hd, cap, B = "bf16", 128, 20000, 16
    nh = g * nkv
    lens = _hn_lens(B, cap, 31 + g, [0, 1, 127, 128, 129, 1000, 8191, 16384, 19999, 20000])
    q = W.normal_tensor((B, nh, hd), 16 + g, 0, dtype)
    kc = nan_padded(B, nkv, cap, hd, lens, 16 + g, 1, dtype)
    vc = nan_padded(B, nkv, cap, hd, lens, 16 + g, 2, dtype)
    want = ref.decode_attention(q.f64, np.nan_to_num(kc.f64), np.nan_to_num(vc.f64), lens)
    ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap, 0) // 4 + 1,
                     dtype=torch.float32, device="cuda")
    n_counters = B * nkv * ((g + 15) // 16)
    gqa.gqa_device_error()
    for call in range(2):
        out = torch.empty((B, nh, hd), dtype=torch.bfloat16, device="cuda")
        gqa.gqa_attn_decode(dev(q), dev(kc), dev(vc), dev_i32(lens), out, ws)
        got = host(out)
        assert np.all(got[0] == 0)
        gate(got[1:], want[1:], dtype, f"keys-as-rows decode, call {call}")
        assert int(ws[:n_counters].view(torch.int32).abs().sum()) == 0
    assert gqa.gqa_device_error() == 0


@pytest.mark.parametrize("long_len", (20000, 8192), ids=["172-tiles", "79-tiles"])
def test_decode_keys_as_rows_many_pieces(long_len):
    """One long sequence among 15 one-key sequences.  20000 keys: 172 tiles
    over the SMs, so the long sequence is cut into pieces of one or two tiles
    on over 100 CTAs, more than the shared-memory merge takes at once (its
    merge runs in rounds over the workspace).  8192 keys: 79 tiles, fewer than
    the SMs, so the tiles are cut over 79 CTAs of one tile and the rest idle."""
    dtype, hd, nh, nkv, cap, B = "bf16", 128, 32, 1, 20000, 16
    lens = np.array([1] * 6 + [long_len] + [1] * 9, dtype=np.int32)
    q = W.normal_tensor((B, nh, hd), 23, 0, dtype)
    kc = nan_padded(B, nkv, cap, hd, lens, 23, 1, dtype)
    vc = nan_padded(B, nkv, cap, hd, lens, 23, 2, dtype)
    want = ref.decode_attention(q.f64, np.nan_to_num(kc.f64), np.nan_to_num(vc.f64), lens)
    gate(host(run_decode(q, kc, vc, lens, nh, dtype)), want, dtype, "keys-as-rows decode, many pieces")


def test_decode_keys_as_rows_degenerate_lengths():
    """The keys-as-rows decode with every length 0 (no tiles anywhere: every
    output row is written as zeros by its CTA) and with lengths past the
    cache (clamped to it and flagged)."""
    dtype, hd, nh, nkv, cap, B = "bf16", 128, 32, 1, 20000, 16
    q = W.normal_tensor((B, nh, hd), 29, 0, dtype)
    zero = np.zeros(B, dtype=np.int32)
    kc = nan_padded(B, nkv, cap, hd, zero, 29, 1, dtype)
    vc = nan_padded(B, nkv, cap, hd, zero, 29, 2, dtype)
    gqa.gqa_device_error()
    out = run_decode(q, kc, vc, zero, nh, dtype)
    assert np.all(host(out) == 0)
    assert gqa.gqa_device_error() == 0
    lens = np.array([cap + 5] + [700] * (B - 1), dtype=np.int32)
    full = np.minimum(lens, cap).astype(np.int32)
    kc = nan_padded(B, nkv, cap, hd, full, 30, 1, dtype)
    vc = nan_padded(B, nkv, cap, hd, full, 30, 2, dtype)
    got = host(run_decode(q, kc, vc, lens, nh, dtype))
    assert gqa.gqa_device_error() & 2
    want = ref.decode_attention(q.f64, np.nan_to_num(kc.f64), np.nan_to_num(vc.f64), full)
    gate(got, want, dtype, "keys-as-rows decode, clamped lengths")


def test_decode_long_cache_uses_workspace_splits():
    """A cache longer than 8 x 2048 keys takes the workspace splits even when
    the split is left to the library."""
    dtype, hd, nh, nkv, cap = "bf16", 128, 8, 1, 20000
    lens = np.array([20000, 12345], dtype=np.int32)
    B = len(lens)
    q = W.normal_tensor((B, nh, hd), 13, 0, dtype)
    kc = nan_padded(B, nkv, cap, hd, lens, 13, 1, dtype)
    vc = nan_padded(B, nkv, cap, hd, lens, 13, 2, dtype)
    want = ref.decode_attention(q.f64, np.nan_to_num(kc.f64), np.nan_to_num(vc.f64), lens)
    gate(host(run_decode(q, kc, vc, lens, nh, dtype)), want, dtype, "long-cache decode")


def paged_inputs(B, nh, nkv, hd, ps, lens, seed, extra_pages=5, min_cap=0):
    """The seeded contiguous decode cache cut into pages of ``ps`` keys, the
    pages shuffled into a pool with ``extra_pages`` NaN-filled pages that no
    table names; table entries past a sequence's last page are -1.  The
    table's width (the logical capacity) covers at least ``min_cap`` keys."""
    cap = -(-max(int(lens.max()), 1, min_cap) // ps) * ps
    max_pages = cap // ps
    q = W.normal_tensor((B, nh, hd), seed, 0, "bf16")
    kc = nan_padded(B, nkv, cap, hd, lens, seed, 1, "bf16")
    vc = nan_padded(B, nkv, cap, hd, lens, seed, 2, "bf16")
    n_pool = B * max_pages + extra_pages
    perm = np.random.default_rng(seed + 1000).permutation(n_pool)      # logical page i -> physical perm[i]

    def cut(c):
        logical = c.store.reshape(B, nkv, max_pages, ps, hd).transpose(0, 2, 1, 3, 4).reshape(-1, nkv, ps, hd)
        pool = np.full((n_pool, nkv, ps, hd), SENTINEL["bf16"], dtype=np.uint16)
        pool[perm[:B * max_pages]] = logical
        return W.Tensor(pool, "bf16")

    table = perm[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    for b in range(B):
        table[b, -(-int(lens[b]) // ps):] = -1
    return q, kc, vc, cut(kc), cut(vc), table, cap


def run_decode_paged(q, kp, vp, table, lens, nh, kv_split=0):
    B, _, hd = q.shape
    nkv, ps = kp.shape[1], kp.shape[2]
    cap = table.shape[1] * ps
    ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap, kv_split) // 4 + 1,
                     dtype=torch.float32, device="cuda")
    out = torch.empty((B, nh, hd), dtype=torch.bfloat16, device="cuda")
    gqa.gqa_attn_decode_paged(dev(q), dev(kp), dev(vp), dev_i32(table), dev_i32(lens), out, ws, kv_split=kv_split)
    return out


@pytest.mark.parametrize("hd,g,nkv,ps", [(128, 8, 1, 64), (128, 4, 2, 128), (64, 48, 1, 64), (64, 2, 4, 256),
                                         (128, 32, 1, 192)])
def test_paged_decode_parity(hd, g, nkv, ps):
    """Decode over shuffled pages against the oracle's paged decode, for the
    automatic split and two fixed ones, and bit for bit against the same
    cache laid out contiguously (only the address of each tile differs)."""
    nh = g * nkv
    lens = np.array([1, 63, 64, 65, 300, 1000, 0, 513, 2000], dtype=np.int32)
    B = len(lens)
    q, kc, vc, kp, vp, table, cap = paged_inputs(B, nh, nkv, hd, ps, lens, 60 + hd + ps)
    want = ref.paged_decode_attention(q.f64, kp.f64, vp.f64, table, lens, ps)
    gqa.gqa_device_error()
    for split in (0, 64, 192):
        got_t = run_decode_paged(q, kp, vp, table, lens, nh, kv_split=split)
        got = host(got_t)
        assert np.all(got[6] == 0)
        keep = lens > 0
        gate(got[keep], want[keep], "bf16", f"paged decode split={split}")
        flat = run_decode(q, kc, vc, lens, nh, "bf16", kv_split=split)
        np.testing.assert_array_equal(bits(got_t), bits(flat))
    assert gqa.gqa_device_error() == 0


@pytest.mark.parametrize("ps", (64, 192))
def test_paged_decode_keys_as_rows(ps):
    """The keys-as-rows decode (B 32, 32 heads on one KV head, up to 8192
    keys) over shuffled pages, its table wide enough (20000 keys) that the
    cluster kernel does not take it: every 64-key half of a 128-key tile is
    mapped to its page (a 192-key page holds one and a half tiles); against
    the oracle's paged decode, and bit for bit against the same keys in a
    contiguous cache of 20000 slots (the same kernel: only the address of
    each tile differs)."""
    hd, g, nkv, B = 128, 32, 1, 32
    nh = g * nkv
    lens = _hn_lens(B, 8192, 77 + ps, [8192, 0, 1, 64, 127, 128, 129, 191, 192, 193, 5000])
    q, kc, vc, kp, vp, table, cap = paged_inputs(B, nh, nkv, hd, ps, lens, 90 + ps, min_cap=20000)
    want = ref.paged_decode_attention(q.f64, kp.f64, vp.f64, table, lens, ps)
    gqa.gqa_device_error()
    got_t = run_decode_paged(q, kp, vp, table, lens, nh)
    got = host(got_t)
    assert np.all(got[1] == 0)
    keep = lens > 0
    gate(got[keep], want[keep], "bf16", f"paged keys-as-rows decode ps={ps}")
    assert kc.shape[2] >= 20000           # the contiguous copy is as wide as the table
    flat = run_decode(q, kc, vc, lens, nh, "bf16")
    np.testing.assert_array_equal(bits(got_t), bits(flat))
    assert gqa.gqa_device_error() == 0


@pytest.mark.parametrize("hd,ps", [(128, 64), (128, 192), (64, 128)])
def test_paged_decode_cluster_kernel(hd, ps):
    """Large paged batches with g > 16 and at most 8 x 2048 keys per
    sequence take the cluster tcgen05 decode (heads as the MMA rows), with
    each 64-key tile mapped to its page: against the oracle's paged decode,
    bit for bit against the same keys in a contiguous cache of the same
    capacity (the same kernel), and with bad table entries flagged and read
    as zeros."""
    g, nkv, B = 32, 1, 32
    nh = g * nkv
    lens = _hn_lens(B, 8192, 55 + ps + hd, [8192, 0, 1, 63, 64, 65, 191, 192, 193, 2048, 5000])
    q, kc, vc, kp, vp, table, cap = paged_inputs(B, nh, nkv, hd, ps, lens, 95 + ps + hd)
    assert cap <= 8 * 2048
    want = ref.paged_decode_attention(q.f64, kp.f64, vp.f64, table, lens, ps)
    gqa.gqa_device_error()
    got_t = run_decode_paged(q, kp, vp, table, lens, nh)
    got = host(got_t)
    assert np.all(got[1] == 0)
    keep = lens > 0
    gate(got[keep], want[keep], "bf16", f"paged cluster decode hd={hd} ps={ps}")
    flat = run_decode(q, kc, vc, lens, nh, "bf16")
    np.testing.assert_array_equal(bits(got_t), bits(flat))
    assert gqa.gqa_device_error() == 0
    # two bad entries: past the pool, and negative, inside the sequences' key ranges
    n_pool = kp.shape[0]
    bad = table.copy()
    bad[0, 3] = n_pool + 11
    bad[5, 0] = -3
    got = host(run_decode_paged(q, kp, vp, bad, lens, nh))
    assert gqa.gqa_device_error() & 8
    zk = np.concatenate([kp.f64, np.zeros((1,) + kp.shape[1:])])
    zv = np.concatenate([vp.f64, np.zeros((1,) + vp.shape[1:])])
    zt = np.where((bad < 0) | (bad >= n_pool), n_pool, bad)
    want = ref.paged_decode_attention(q.f64, zk, zv, zt, lens, ps)
    gate(got[keep], want[keep], "bf16", "paged cluster decode, zero-read pages")


def test_paged_decode_shared_pages():
    """Two sequences whose tables name the same physical pages (a shared
    prompt prefix) attend over the same keys: identical queries give
    identical outputs."""
    hd, nh, nkv, ps = 128, 16, 2, 64
    lens = np.array([700, 700], dtype=np.int32)
    q, kc, vc, kp, vp, table, cap = paged_inputs(2, nh, nkv, hd, ps, lens, 71)
    table[1] = table[0]
    qs = W.Tensor(np.ascontiguousarray(np.broadcast_to(q.store[:1], q.store.shape)), "bf16")
    out = run_decode_paged(qs, kp, vp, table, lens, nh)
    got = bits(out)
    np.testing.assert_array_equal(got[0], got[1])
    want = ref.paged_decode_attention(qs.f64, kp.f64, vp.f64, table, lens, ps)
    gate(host(out), want, "bf16", "shared pages")


def test_paged_decode_bad_table_entry_flags_and_reads_zeros():
    """A table entry outside the page pool raises the page-range bit; its
    keys read as zeros (score 0, value 0), which the oracle reproduces with a
    zero page in that slot."""
    hd, nh, nkv, ps = 64, 8, 1, 64
    lens = np.array([256, 130], dtype=np.int32)
    q, kc, vc, kp, vp, table, cap = paged_inputs(2, nh, nkv, hd, ps, lens, 72)
    n_pool = kp.shape[0]
    bad = table.copy()
    bad[0, 1] = n_pool + 3
    bad[1, 0] = -7
    gqa.gqa_device_error()
    got = host(run_decode_paged(q, kp, vp, bad, lens, nh))
    assert gqa.gqa_device_error() & 8
    zk = np.concatenate([kp.f64, np.zeros((1,) + kp.shape[1:])])
    zv = np.concatenate([vp.f64, np.zeros((1,) + vp.shape[1:])])
    zt = np.where((bad < 0) | (bad >= n_pool), n_pool, bad)      # bad entries -> the zero page
    want = ref.paged_decode_attention(q.f64, zk, zv, zt, lens, ps)
    gate(got, want, "bf16", "zero-read pages")


def test_injected_launch_failure_leaves_the_library_usable():
    """A failure injected on the host surfaces as GQAError (launch failed)
    and launches nothing; the next call runs and gives the same bits."""
    dtype, hd, nh, nkv, cap = "bf16", 128, 8, 2, 256
    lens = np.array([256, 100], dtype=np.int32)
    q = W.normal_tensor((2, nh, hd), 15, 0, dtype)
    kc = nan_padded(2, nkv, cap, hd, lens, 15, 1, dtype)
    vc = nan_padded(2, nkv, cap, hd, lens, 15, 2, dtype)
    first = bits(run_decode(q, kc, vc, lens, nh, dtype))
    n0 = gqa.gqa_launch_count()
    gqa.gqa_debug_inject_launch_failures(1)
    try:
        with pytest.raises(gqa.GQAError) as e:
            run_decode(q, kc, vc, lens, nh, dtype)
        assert e.value.status == -6
        assert gqa.gqa_launch_count() == n0
    finally:
        gqa.gqa_debug_inject_launch_failures(0)
    np.testing.assert_array_equal(bits(run_decode(q, kc, vc, lens, nh, dtype)), first)


def test_decode_zero_and_clamped_lengths():
    dtype, hd, nh, nkv, cap = "bf16", 64, 4, 2, 128
    lens = np.array([0, 128, 5], dtype=np.int32)
    q = W.normal_tensor((3, nh, hd), 9, 0, dtype)
    kc = nan_padded(3, nkv, cap, hd, lens, 9, 1, dtype)
    vc = nan_padded(3, nkv, cap, hd, lens, 9, 2, dtype)
    gqa.gqa_device_error()
    out = run_decode(q, kc, vc, lens, nh, dtype)
    assert gqa.gqa_device_error() == 0
    got = host(out)
    assert np.all(got[0] == 0)
    want = ref.decode_attention(q.f64, np.nan_to_num(kc.f64), np.nan_to_num(vc.f64), lens)
    gate(got[1:], want[1:], dtype, "decode lens")
    # a length above cap is clamped and flagged
    over = run_decode(q, kc, vc, np.array([0, 500, 5], dtype=np.int32), nh, dtype)
    assert gqa.gqa_device_error() & 2
    gate(host(over)[1:], want[1:], dtype, "clamped")


def test_prefill_last_row_equals_decode_on_gpu():
    dtype, B, nh, nkv, S, hd = "bf16", 2, 8, 2, 77, 128
    lens = np.array([S, S], dtype=np.int32)
    q, kc, vc = attn_inputs(B, nh, nkv, S, hd, S, lens, dtype, seed=5)
    out = torch.empty((B, S, nh, hd), dtype=torch.bfloat16, device="cuda")
    gqa.gqa_attn_prefill(dev(q), dev(kc), dev(vc), dev_i32(lens), True, out)
    qd = W.Tensor(np.ascontiguousarray(q.store[:, :, -1]), "bf16")
    d = run_decode(qd, kc, vc, lens, nh, dtype)
    want = ref.decode_attention(qd.f64, kc.f64, vc.f64, lens)
    gate(host(d), want, dtype, "decode")
    gate(host(out)[:, -1], want, dtype, "prefill last row")


# --------------------------------------------------------------------------
# MHA -> GQA weight transform (mean pooling of each group's KV projections)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("dtype,nh,nkv,hd,D", [
    ("bf16", 32, 8, 128, 512), ("bf16", 32, 1, 64, 264), ("bf16", 12, 4, 32, 8), ("bf16", 6, 6, 64, 136),
    ("f32", 12, 4, 64, 100), ("f32", 6, 2, 128, 36),
])
def test_meanpool_kv_heads_parity(dtype, nh, nkv, hd, D):
    w = W.normal_tensor((3 * nh * hd, D), 15, nh + nkv, dtype, std=0.02)
    out = torch.empty(((nh + 2 * nkv) * hd, D), dtype=TORCH_DT[dtype], device="cuda")
    gqa.gqa_meanpool_kv_heads(dev(w), nh, nkv, hd, out)
    want = ref.meanpool_kv_projection(w.f64, nh, nkv, hd)
    raw = w.store.view(np.uint16 if dtype == "bf16" else np.uint32)
    assert np.array_equal(bits(out)[: nh * hd], raw[: nh * hd])               # query rows copied bit for bit
    if nkv == nh:
        assert np.array_equal(bits(out), raw)                                 # n_kv_heads = n_heads: a copy
    gate(host(out), want, dtype, "mean-pooled W_qkv")


def test_meanpool_of_replicated_kv_heads_is_exact():
    """An MHA weight whose KV heads repeat each GQA head g times (g a power of
    two) pools back to the GQA weight bit for bit."""
    nh, nkv, hd, D = 16, 4, 64, 128
    g = nh // nkv
    w_gqa = W.normal_tensor(((nh + 2 * nkv) * hd, D), 16, 0, "bf16", std=0.02)
    s = w_gqa.store
    kv = [s[nh * hd + k * nkv * hd: nh * hd + (k + 1) * nkv * hd].reshape(nkv, hd, D) for k in (0, 1)]
    mha = np.concatenate([s[: nh * hd]] + [np.repeat(t, g, axis=0).reshape(nh * hd, D) for t in kv])
    out = torch.empty(((nh + 2 * nkv) * hd, D), dtype=torch.bfloat16, device="cuda")
    gqa.gqa_meanpool_kv_heads(dev(W.Tensor(np.ascontiguousarray(mha), "bf16")), nh, nkv, hd, out)
    assert np.array_equal(bits(out), s)
