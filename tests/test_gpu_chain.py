"""Dependent launches: every kernel is launched so that it may start while
the kernel before it on the stream is still running, and waits for it
(griddepcontrol.wait) before its first access to global memory.  The layer's
chain of calls (projection -> prefill -> output projection, then one decode
step through the same three) is run twice on one stream: back to back, with
nothing between the library's launches, and with the stream synchronised
after every call.  Both runs must give the same bits in every output, and
the back-to-back run must agree with the oracle on sampled rows."""
import numpy as np
import pytest
import torch

import mqa_attention_qkv_b200 as gqa
import workloads as W
from oracle import gqa_ref as ref
from tests._helpers import bits, dev, dev_i32, gate, host

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _chain(bufs, sh, sync):
    """Run the layer step on the buffers in ``bufs``; synchronise after every
    call when ``sync``."""
    nh, nkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim
    b = bufs
    calls = [
        lambda: gqa.qkv_rope_project(b["x"], b["w"], b["pos"], nh, nkv, hd, sh.rope_theta, b["q"], b["kc"], b["vc"]),
        lambda: gqa.gqa_attn_prefill(b["q"], b["kc"], b["vc"], b["lens"], True, b["o"]),
        lambda: gqa.gqa_o_proj_residual(b["o"], b["w_o"], b["y"], residual=b["x"]),
        lambda: gqa.qkv_rope_project(b["xd"], b["w"], b["posd"], nh, nkv, hd, sh.rope_theta, b["qd"], b["kc"],
                                     b["vc"]),
        lambda: gqa.gqa_attn_decode(b["qd"].view(b["qd"].shape[0], nh, hd), b["kc"], b["vc"], b["lensd"], b["od"],
                                    b["ws"]),
        lambda: gqa.gqa_o_proj_residual(b["od"].view(b["od"].shape[0], 1, nh, hd), b["w_o"], b["yd"],
                                        residual=b["xd"]),
    ]
    for c in calls:
        c()
        if sync:
            torch.cuda.synchronize()
    torch.cuda.synchronize()


def _buffers(sh, B, S, seed):
    nh, nkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim
    cap = S + 1
    x, w, pos = W.layer_inputs(sh, B, S, seed=seed, dtype="bf16")
    xd = W.hidden_states(sh, B, 1, seed=seed, stream=1, dtype="bf16")
    bufs = {
        "x": dev(x), "w": dev(w), "pos": dev_i32(pos), "w_o": dev(W.output_weight(sh, seed, "bf16")),
        "xd": dev(xd), "posd": dev_i32(np.full((B, 1), S, dtype=np.int32)),
        "lens": dev_i32(np.full(B, S)), "lensd": dev_i32(np.full(B, S + 1)),
        "kc": torch.zeros((B, nkv, cap, hd), dtype=BF, device="cuda"),
        "vc": torch.zeros((B, nkv, cap, hd), dtype=BF, device="cuda"),
        "q": torch.empty((B, nh, S, hd), dtype=BF, device="cuda"),
        "o": torch.empty((B, S, nh, hd), dtype=BF, device="cuda"),
        "y": torch.empty((B, S, sh.hidden), dtype=BF, device="cuda"),
        "qd": torch.empty((B, nh, 1, hd), dtype=BF, device="cuda"),
        "od": torch.empty((B, nh, hd), dtype=BF, device="cuda"),
        "yd": torch.empty((B, 1, sh.hidden), dtype=BF, device="cuda"),
        "ws": torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap), dtype=torch.uint8,
                          device="cuda"),
    }
    return bufs, (x, w, pos, xd)


@pytest.mark.parametrize("bs", [(2, 200), (4, 2048)], ids=lambda t: f"{t[0]}x{t[1]}")
def test_back_to_back_layer_step_matches_synchronised_calls(bs):
    wl = W.TINYLLAMA_PREFILL
    sh = wl.shape
    B, S = bs
    outs = ("q", "kc", "vc", "o", "y", "qd", "od", "yd")
    got = {}
    for sync in (True, False):
        bufs, raw = _buffers(sh, B, S, wl.seed)
        torch.cuda.synchronize()
        _chain(bufs, sh, sync)
        got[sync] = {k: bits(bufs[k]) for k in outs}
    for k in outs:
        np.testing.assert_array_equal(got[False][k], got[True][k], err_msg=f"{k}: back to back differs")
    assert gqa.gqa_device_error() == 0
    # the back-to-back decode step against the oracle (bf16 between calls, as the library stores it)
    x, w, pos, xd = raw
    nh, nkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim
    z = np.zeros((B, nkv, S + 1, hd))
    rb = ref.round_bf16
    _, kc_r, vc_r = ref.qkv_rope_project(x.f64, w.f64, pos, nh, nkv, hd, sh.rope_theta, z, z)
    qd_r, kc_r, vc_r = ref.qkv_rope_project(xd.f64, w.f64, np.full((B, 1), S, dtype=np.int32), nh, nkv, hd,
                                            sh.rope_theta, kc_r, vc_r)
    od_r = ref.decode_attention(rb(qd_r[:, :, 0]), rb(kc_r), rb(vc_r), np.full(B, S + 1))
    gate(host(bufs["od"]), od_r, "bf16", "back-to-back decode step")
