"""The attention layer's output projection with the residual add
(gqa_o_proj_residual) on the GPU, against the float64 oracle's
``output_projection``: every kernel path (128-token tensor-core tiles, the
few-token cluster-split tiles, SIMT), ragged token counts and widths, no
residual / a separate one / in place, and the whole layer chained at the
TinyLlama and MQA-generation shapes."""
import numpy as np
import pytest
import torch

import mqa_attention_qkv_b200 as gqa
import workloads as W
from oracle import gqa_ref as ref
from tests._helpers import dev, dev_i32, gate, host

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _inputs(seed, T, nh, hd, hidden, dtype):
    attn = W.normal_tensor((T, nh, hd), seed, 0, dtype)
    w_o = W.normal_tensor((hidden, nh * hd), seed, 1, dtype, std=0.02)
    res = W.normal_tensor((T, hidden), seed, 2, dtype)
    return attn, w_o, res


CASES = [
    # T, n_heads, head_dim, hidden (T <= 64: the W-streaming kernel when nh*hd % 64 == 0 and hidden % 16 == 0,
    # else the cluster-split tensor-core kernel: (13, 5, 32, 264), (33, 8, 128, 1032), (40, 8, 64, 2056))
    (1, 32, 64, 2048), (8, 32, 64, 2048), (13, 5, 32, 264), (33, 8, 128, 1032), (64, 32, 64, 2048),
    (40, 8, 64, 2056), (20, 6, 32, 1040),
    (8, 48, 128, 6144),                               # MQA generation step shape
    (65, 32, 64, 2048), (200, 5, 32, 264), (300, 8, 128, 1032), (1000, 16, 64, 1024),
    (4000, 16, 64, 1536),                             # 192 tiles: the last wave's 44 as 88 half-width tiles
    (6000, 8, 64, 904),                               # split last wave with a ragged N: a half tile of 8 columns
]


@pytest.mark.parametrize("mode", ["none", "residual", "in_place"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "T{}-nh{}-hd{}-N{}".format(*c))
def test_o_proj_parity(case, mode):
    T, nh, hd, hidden = case
    attn, w_o, res = _inputs(100 + T + nh, T, nh, hd, hidden, "bf16")
    a, w = dev(attn), dev(w_o)
    want = ref.output_projection(attn.f64, w_o.f64, None if mode == "none" else res.f64)
    if mode == "in_place":
        out = dev(res)
        gqa.gqa_o_proj_residual(a, w, out, residual=out)
    else:
        out = torch.full((T, hidden), float("nan"), dtype=BF, device="cuda")
        gqa.gqa_o_proj_residual(a, w, out, residual=dev(res) if mode == "residual" else None)
    torch.cuda.synchronize()
    gate(host(out), want, "bf16", f"o_proj {case} {mode}")


def test_o_proj_fp32_and_unaligned_width_take_the_simt_path():
    # float32 (the tiny fp32 layer's widths) and a bf16 width that is not a multiple of 8
    for T, nh, hd, hidden, dt in ((128, 8, 32, 256, "f32"), (70, 4, 32, 100, "bf16"), (5, 4, 64, 36, "bf16")):
        attn, w_o, res = _inputs(7 + hidden, T, nh, hd, hidden, dt)
        out = torch.full((T, hidden), float("nan"), dtype=BF if dt == "bf16" else torch.float32, device="cuda")
        gqa.gqa_o_proj_residual(dev(attn), dev(w_o), out, residual=dev(res))
        torch.cuda.synchronize()
        gate(host(out), ref.output_projection(attn.f64, w_o.f64, res.f64), dt, f"o_proj simt {dt} N{hidden}")


def test_o_proj_writes_nothing_outside_out():
    T, nh, hd, hidden = 40, 8, 64, 520
    attn, w_o, res = _inputs(3, T, nh, hd, hidden, "bf16")
    big = torch.full((T * hidden + 4096,), 7.0, dtype=BF, device="cuda")
    out = big[2048:2048 + T * hidden].view(T, hidden)
    gqa.gqa_o_proj_residual(dev(attn), dev(w_o), out, residual=dev(res))
    torch.cuda.synchronize()
    assert torch.all(big[:2048] == 7.0) and torch.all(big[2048 + T * hidden:] == 7.0)
    gate(host(out), ref.output_projection(attn.f64, w_o.f64, res.f64), "bf16", "o_proj canaries")


def test_o_proj_empty_batch_is_a_noop():
    out = torch.zeros((0, 64), dtype=BF, device="cuda")
    gqa.gqa_o_proj_residual(torch.zeros((0, 2, 32), dtype=BF, device="cuda"),
                            torch.zeros((64, 64), dtype=BF, device="cuda"), out)


@pytest.mark.parametrize("bs", [(2, 96), (4, 2048)], ids=lambda t: f"{t[0]}x{t[1]}")
def test_tinyllama_whole_layer(bs):
    """Projection -> causal prefill -> output projection + residual, then one
    decode step through the same layer, at the TinyLlama shape; sampled
    tokens of the full-size batch against the oracle's chain (q/K/V and the
    attention output stored in bf16 between calls)."""
    wl = W.TINYLLAMA_PREFILL
    sh = wl.shape
    B, S = bs
    nh, nkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim
    cap = S + 1
    x, w, pos = W.layer_inputs(sh, B, S, seed=wl.seed, dtype="bf16")
    w_o = W.output_weight(sh, wl.seed, "bf16")
    xd = W.hidden_states(sh, B, 1, seed=wl.seed, stream=1, dtype="bf16")
    wdev, wodev = dev(w), dev(w_o)
    kc = torch.zeros((B, nkv, cap, hd), dtype=BF, device="cuda")
    vc = torch.zeros_like(kc)
    q = torch.empty((B, nh, S, hd), dtype=BF, device="cuda")
    o = torch.empty((B, S, nh, hd), dtype=BF, device="cuda")
    y = torch.empty((B, S, sh.hidden), dtype=BF, device="cuda")
    xdev = dev(x)
    gqa.qkv_rope_project(xdev, wdev, dev_i32(pos), nh, nkv, hd, sh.rope_theta, q, kc, vc)
    gqa.gqa_attn_prefill(q, kc, vc, dev_i32(np.full(B, S)), True, o)
    gqa.gqa_o_proj_residual(o, wodev, y, residual=xdev)
    qd = torch.empty((B, nh, 1, hd), dtype=BF, device="cuda")
    posd = np.full((B, 1), S, dtype=np.int32)
    xddev = dev(xd)
    gqa.qkv_rope_project(xddev, wdev, dev_i32(posd), nh, nkv, hd, sh.rope_theta, qd, kc, vc)
    od = torch.empty((B, nh, hd), dtype=BF, device="cuda")
    ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap), dtype=torch.uint8, device="cuda")
    gqa.gqa_attn_decode(qd.view(B, nh, hd), kc, vc, dev_i32(np.full(B, S + 1)), od, ws)
    yd = torch.empty((B, 1, sh.hidden), dtype=BF, device="cuda")
    gqa.gqa_o_proj_residual(od.view(B, 1, nh, hd), wodev, yd, residual=xddev)
    torch.cuda.synchronize()

    rb = ref.round_bf16
    z = np.zeros((B, nkv, cap, hd))
    q_r, kc_r, vc_r = ref.qkv_rope_project(x.f64, w.f64, pos, nh, nkv, hd, sh.rope_theta, z, z)
    qd_r, kc_r, vc_r = ref.qkv_rope_project(xd.f64, w.f64, posd, nh, nkv, hd, sh.rope_theta, kc_r, vc_r)
    r = np.random.default_rng(5)
    toks = sorted({(int(r.integers(B)), int(r.integers(S))) for _ in range(24)} | {(0, 0), (B - 1, S - 1)})
    rows = [(b, h, s) for b, s in toks for h in range(nh)]
    o_rows = ref.prefill_attention(rb(q_r), rb(kc_r), rb(vc_r), np.full(B, S), True, rows=rows)
    o_tok = rb(np.asarray(o_rows).reshape(len(toks), nh, hd))        # attention output stored in bf16
    y_r = ref.output_projection(o_tok, w_o.f64, np.stack([x.f64[b, s] for b, s in toks]))
    yh = host(y)
    gate(np.stack([yh[b, s] for b, s in toks]), y_r, "bf16", "layer output (prefill)")
    od_r = ref.decode_attention(rb(qd_r[:, :, 0]), rb(kc_r), rb(vc_r), np.full(B, S + 1))
    yd_r = ref.output_projection(rb(od_r)[:, None], w_o.f64, xd.f64)
    gate(host(yd), yd_r, "bf16", "layer output (decode step)")


def test_mqa_generation_step_with_output_projection():
    """One decode step of the MQA generation shape (B 8, 48 heads, hidden
    6144) through projection, decode and output projection + residual."""
    wl = W.MQA_GENERATE
    sh, e = wl.shape, wl.extra
    B, cap = e["batch"], e["cap"]
    nh, nkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim
    L = 300
    w = W.weight(sh, wl.seed, "bf16")
    w_o = W.output_weight(sh, wl.seed, "bf16")
    x = W.hidden_states(sh, B, L, wl.seed, 0, "bf16")
    pos = np.broadcast_to(np.arange(L, dtype=np.int32), (B, L)).copy()
    wdev = dev(w)
    kc = torch.zeros((B, nkv, cap, hd), dtype=BF, device="cuda")
    vc = torch.zeros_like(kc)
    q = torch.empty((B, nh, L, hd), dtype=BF, device="cuda")
    gqa.qkv_rope_project(dev(x), wdev, dev_i32(pos), nh, nkv, hd, sh.rope_theta, q, kc, vc)
    qt = q[:, :, L - 1].contiguous()
    ot = torch.empty((B, nh, hd), dtype=BF, device="cuda")
    ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap), dtype=torch.uint8, device="cuda")
    gqa.gqa_attn_decode(qt, kc, vc, dev_i32(np.full(B, L)), ot, ws)
    xt = dev(x)[:, L - 1].contiguous()
    y = xt.clone()
    gqa.gqa_o_proj_residual(ot.view(B, nh, hd), dev(w_o), y, residual=y)   # in place on the residual stream
    torch.cuda.synchronize()
    rb = ref.round_bf16
    z = np.zeros((B, nkv, cap, hd))
    q_r, kc_r, vc_r = ref.qkv_rope_project(x.f64, w.f64, pos, nh, nkv, hd, sh.rope_theta, z, z)
    o_r = ref.decode_attention(rb(q_r[:, :, L - 1]), rb(kc_r), rb(vc_r), np.full(B, L))
    gate(host(ot), o_r, "bf16", "decode")
    y_r = ref.output_projection(rb(o_r), w_o.f64, x.f64[:, L - 1])
    gate(host(y), y_r, "bf16", "layer output")
