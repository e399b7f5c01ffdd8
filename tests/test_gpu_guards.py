"""Canaries around every output buffer: each call writes its outputs and
nothing next to them.  Outputs are slices of larger NaN-filled buffers; the
guard regions before and after each slice must still be NaN after the call.
Ragged shapes put the kernels' tile tails right at the buffer edges."""
import numpy as np
import pytest
import torch

import mqa_attention_qkv_b200 as gqa
import workloads as W
from tests._helpers import dev, dev_i32

pytestmark = pytest.mark.gpu

GUARD = 4096   # elements on each side (8 KB of bf16: 16-byte aligned slices)


def guarded(shape, dtype=torch.bfloat16, fill=float("nan")):
    n = int(np.prod(shape))
    buf = torch.full((GUARD + n + GUARD,), fill, dtype=dtype, device="cuda")
    return buf, buf[GUARD:GUARD + n].view(shape)


def assert_guards(buf, shape, what, fill=None):
    """Guards still hold NaN (float buffers) or `fill` (byte buffers)."""
    n = int(np.prod(shape))
    torch.cuda.synchronize()
    for g in (buf[:GUARD], buf[GUARD + n:]):
        ok = torch.isnan(g.float()).all() if fill is None else (g == fill).all()
        assert ok, f"{what}: a write landed outside the buffer"


def cache(B, nkv, cap, hd, lens, seed, tid):
    return dev(W.decode_cache(seed, tid, B, nkv, cap, hd, lens))


@pytest.mark.parametrize("B,S,hidden,nh,nkv,hd,cap", [(1, 65, 2048, 32, 4, 64, 80), (3, 130, 256, 8, 1, 128, 200),
                                                      (4, 1, 2048, 32, 4, 64, 8), (2, 37, 100, 4, 2, 64, 40)])
def test_projection_writes_only_q_and_its_cache_rows(B, S, hidden, nh, nkv, hd, cap):
    x = dev(W.normal_tensor((B, S, hidden), 1, 0, "bf16"))
    w = dev(W.normal_tensor(((nh + 2 * nkv) * hd, hidden), 1, 1, "bf16", std=0.02))
    pos = dev_i32(np.tile(np.arange(S, dtype=np.int32), (B, 1)))
    qb, q = guarded((B, nh, S, hd))
    kb, kc = guarded((B, nkv, cap, hd))
    vb, vc = guarded((B, nkv, cap, hd))
    gqa.qkv_rope_project(x, w, pos, nh, nkv, hd, 10000.0, q, kc, vc)
    for b_, shp, name in ((qb, (B, nh, S, hd), "q"), (kb, (B, nkv, cap, hd), "k cache"),
                          (vb, (B, nkv, cap, hd), "v cache")):
        assert_guards(b_, shp, f"projection {name}")
    assert not torch.isnan(q.float()).any()


@pytest.mark.parametrize("hd", [64, 128])
def test_prefill_writes_only_its_output(hd):
    B, nh, nkv, S = 3, 8, 2, 129
    lens = np.array([129, 129, 129], dtype=np.int32)
    q = dev(W.normal_tensor((B, nh, S, hd), 2, 0, "bf16"))
    kc, vc = cache(B, nkv, S, hd, lens, 2, 1), cache(B, nkv, S, hd, lens, 2, 2)
    ob, o = guarded((B, S, nh, hd))
    gqa.gqa_attn_prefill(q, kc, vc, dev_i32(lens), True, o)
    assert_guards(ob, (B, S, nh, hd), f"prefill hd {hd}")
    assert not torch.isnan(o.float()).any()


def test_packed_prefill_writes_only_its_output():
    nh, nkv, hd = 8, 2, 64
    seq = np.array([1, 129, 0, 300], dtype=np.int32)
    cu = dev_i32(np.concatenate([[0], np.cumsum(seq)]))
    tot = int(seq.sum())
    q = dev(W.normal_tensor((tot, nh, hd), 3, 0, "bf16"))
    k = dev(W.normal_tensor((tot, nkv, hd), 3, 1, "bf16"))
    v = dev(W.normal_tensor((tot, nkv, hd), 3, 2, "bf16"))
    ob, o = guarded((tot, nh, hd))
    gqa.gqa_attn_prefill_varlen(q, k, v, cu, cu, int(seq.max()), True, o)
    assert_guards(ob, (tot, nh, hd), "packed prefill")
    assert not torch.isnan(o.float()).any()


@pytest.mark.parametrize("B,nh,nkv,hd,cap,split", [(8, 48, 1, 128, 1040, 0), (8, 48, 1, 128, 1040, 64),
                                                    (32, 48, 1, 64, 8192, 0), (5, 8, 8, 32, 300, 0),
                                                    (16, 48, 1, 128, 20000, 0), (16, 128, 2, 128, 20000, 0)],
                         ids=["cluster", "workspace", "tcgen05", "simt-hd32", "keys-as-rows-g48", "keys-as-rows-g64"])
def test_decode_writes_only_its_output(B, nh, nkv, hd, cap, split):
    lens = np.clip(W.ragged_lengths(B, 1, cap, 4), 1, cap).astype(np.int32)
    q = dev(W.normal_tensor((B, nh, hd), 4, 0, "bf16"))
    kc, vc = cache(B, nkv, cap, hd, lens, 4, 1), cache(B, nkv, cap, hd, lens, 4, 2)
    ws_bytes = gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap, split)
    ws_bytes = (ws_bytes + 15) // 16 * 16
    wb, ws = guarded((ws_bytes,), torch.uint8, fill=0xA5)
    ws.zero_()
    ob, o = guarded((B, nh, hd))
    gqa.gqa_attn_decode(q, kc, vc, dev_i32(lens), o, ws, kv_split=split)
    assert_guards(ob, (B, nh, hd), "decode output")
    assert_guards(wb, (ws_bytes,), "decode workspace", fill=0xA5)
    assert not torch.isnan(o.float()).any()


def test_meanpool_writes_only_its_output():
    nh, nkv, hd, D = 32, 8, 128, 520
    w = dev(W.normal_tensor((3 * nh * hd, D), 5, 0, "bf16", std=0.02))
    ob, o = guarded(((nh + 2 * nkv) * hd, D))
    gqa.gqa_meanpool_kv_heads(w, nh, nkv, hd, o)
    assert_guards(ob, ((nh + 2 * nkv) * hd, D), "mean-pool")
    assert not torch.isnan(o.float()).any()
