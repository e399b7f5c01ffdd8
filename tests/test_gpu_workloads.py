"""The five workloads at full size on the GPU, through the C ABI, against the
float64 oracle.  The tiny fp32 layer is compared element by element; the
larger ones on sampled rows that the oracle computes one by one (the oracle's
inputs are regenerated from the same seeded streams, never read back from the
GPU's outputs).

Workloads (see ``workloads``): tiny fp32 GQA layer; TinyLlama-1.1B-shaped
prefill at 1x128, 8x512 and 4x2048 plus one decode step (the benchmark's
step); Llama-2-7B-shaped batched decode with MHA/GQA/MQA caches; the batch-8,
prompt-16, 1024-step MQA generation loop; 8K-token prefill with outlier
channels, causal and not.
"""
import numpy as np
import pytest
import torch

import mqa_attention_qkv_b200 as gqa
import workloads as W
from oracle import gqa_ref as ref
from tests._helpers import dev, dev_i32, gate, host

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _zeros_cache(B, nkv, cap, hd, dt=BF):
    return torch.zeros((B, nkv, cap, hd), dtype=dt, device="cuda")


def test_tiny_fp32_layer_full():
    wl = W.TINY_FP32
    sh = wl.shape
    B, S = wl.batch_seq[0]
    x, w, pos = W.layer_inputs(sh, B, S, seed=wl.seed, dtype="f32")
    kc = _zeros_cache(B, sh.n_kv_heads, S, sh.head_dim, torch.float32)
    vc = torch.zeros_like(kc)
    q = torch.empty((B, sh.n_heads, S, sh.head_dim), dtype=torch.float32, device="cuda")
    o = torch.empty((B, S, sh.n_heads, sh.head_dim), dtype=torch.float32, device="cuda")
    gqa.qkv_rope_project(dev(x), dev(w), dev_i32(pos), sh.n_heads, sh.n_kv_heads, sh.head_dim,
                         sh.rope_theta, q, kc, vc)
    gqa.gqa_attn_prefill(q, kc, vc, dev_i32(np.full(B, S)), True, o)
    z = np.zeros((B, sh.n_kv_heads, S, sh.head_dim))
    q_r, kc_r, vc_r = ref.qkv_rope_project(x.f64, w.f64, pos, sh.n_heads, sh.n_kv_heads, sh.head_dim,
                                           sh.rope_theta, z, z)
    o_r = ref.prefill_attention(q_r, kc_r, vc_r, np.full(B, S), causal=True)
    gate(host(q), q_r, "f32", "q")
    gate(host(kc), kc_r, "f32", "k cache")
    gate(host(vc), vc_r, "f32", "v cache")
    gate(host(o), o_r, "f32", "attention")


@pytest.mark.parametrize("bs", W.TINYLLAMA_PREFILL.batch_seq, ids=lambda t: f"{t[0]}x{t[1]}")
def test_tinyllama_prefill_and_decode_step(bs):
    wl = W.TINYLLAMA_PREFILL
    sh = wl.shape
    B, S = bs
    nh, nkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim
    cap = S + 64
    x, w, pos = W.layer_inputs(sh, B, S, seed=wl.seed, dtype="bf16")
    xd = W.hidden_states(sh, B, 1, seed=wl.seed, stream=1, dtype="bf16")
    kc, vc = _zeros_cache(B, nkv, cap, hd), _zeros_cache(B, nkv, cap, hd)
    q = torch.empty((B, nh, S, hd), dtype=BF, device="cuda")
    o = torch.empty((B, S, nh, hd), dtype=BF, device="cuda")
    wd = dev(w)
    gqa.qkv_rope_project(dev(x), wd, dev_i32(pos), nh, nkv, hd, sh.rope_theta, q, kc, vc)
    gqa.gqa_attn_prefill(q, kc, vc, dev_i32(np.full(B, S)), True, o)
    qd = torch.empty((B, nh, 1, hd), dtype=BF, device="cuda")
    posd = np.full((B, 1), S, dtype=np.int32)
    gqa.qkv_rope_project(dev(xd), wd, dev_i32(posd), nh, nkv, hd, sh.rope_theta, qd, kc, vc)
    od = torch.empty((B, nh, hd), dtype=BF, device="cuda")
    ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap), dtype=torch.uint8, device="cuda")
    gqa.gqa_attn_decode(qd.view(B, nh, hd), kc, vc, dev_i32(np.full(B, S + 1)), od, ws)
    torch.cuda.synchronize()

    z = np.zeros((B, nkv, cap, hd))
    q_r, kc_r, vc_r = ref.qkv_rope_project(x.f64, w.f64, pos, nh, nkv, hd, sh.rope_theta, z, z)
    qd_r, kc_r, vc_r = ref.qkv_rope_project(xd.f64, w.f64, posd, nh, nkv, hd, sh.rope_theta, kc_r, vc_r)
    r = np.random.default_rng(0)
    rows = [(int(r.integers(B)), int(r.integers(nh)), int(r.integers(S))) for _ in range(96)]
    rows += [(0, 0, 0), (B - 1, nh - 1, S - 1), (0, nh - 1, S - 1)]
    qh = host(q)
    gate(np.stack([qh[b, h, s] for b, h, s in rows]), np.stack([q_r[b, h, s] for b, h, s in rows]), "bf16", "q")
    kh, vh = host(kc), host(vc)
    slots = sorted(set(int(s) for _, _, s in rows)) + [S]
    gate(kh[:, :, slots], kc_r[:, :, slots], "bf16", "k cache")
    gate(vh[:, :, slots], vc_r[:, :, slots], "bf16", "v cache")
    # attention reads the bf16 q/K/V that the projection stored
    rq, rk, rv = ref.round_bf16(q_r), ref.round_bf16(kc_r), ref.round_bf16(vc_r)
    o_r = ref.prefill_attention(rq, rk, rv, np.full(B, S), True, rows=rows)
    oh = host(o)
    gate(np.stack([oh[b, s, h] for b, h, s in rows]), o_r, "bf16", "prefill attention")
    od_r = ref.decode_attention(ref.round_bf16(qd_r[:, :, 0]), rk, rv, np.full(B, S + 1))
    gate(host(od), od_r, "bf16", "decode step")


@pytest.mark.parametrize("nkv", W.LLAMA2_DECODE.extra["n_kv_heads_cases"])
def test_llama2_decode_full(nkv):
    wl = W.LLAMA2_DECODE
    e = wl.extra
    B, nh, hd, cap = e["batch"], wl.shape.n_heads, wl.shape.head_dim, e["cap"]
    lens = W.ragged_lengths(B, e["kv_lo"], e["kv_hi"], wl.seed)
    q = W.normal_tensor((B, nh, hd), wl.seed, 0, "bf16")
    kc = W.decode_cache(wl.seed, 1, B, nkv, cap, hd, lens)
    kd = dev(kc)
    del kc
    vc = W.decode_cache(wl.seed, 2, B, nkv, cap, hd, lens)
    vd = dev(vc)
    del vc
    ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, nh, hd), dtype=BF, device="cuda")
    gqa.gqa_attn_decode(dev(q), kd, vd, dev_i32(lens), out, ws)
    got = host(out)
    r = np.random.default_rng(1)
    pairs = [(int(r.integers(B)), int(r.integers(nh))) for _ in range(40)]
    pairs += [(int(np.argmax(lens)), 0), (int(np.argmin(lens)), nh - 1)]
    g = nh // nkv
    want, have = [], []
    for b, h in pairs:
        L = int(lens[b])
        j = h // g
        K = W.bf16_to_f32(W.bf16_bits(W.cache_rows(wl.seed, 1, b, j, L, hd))).astype(np.float64)
        V = W.bf16_to_f32(W.bf16_bits(W.cache_rows(wl.seed, 2, b, j, L, hd))).astype(np.float64)
        o, _ = ref.attend_row(q.f64[b, h], K, V)
        want.append(o)
        have.append(got[b, h])
    gate(np.stack(have), np.stack(want), "bf16", f"decode nkv={nkv}")
    assert np.all(np.isfinite(got))


def test_mqa_generation_loop_full():
    """Prompt of 16 then 1024 one-token steps, the cache grown in place."""
    wl = W.MQA_GENERATE
    sh, e = wl.shape, wl.extra
    B, P, T, cap = e["batch"], e["prompt"], e["steps"], e["cap"]
    nh, nkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim
    w = W.weight(sh, wl.seed, "bf16")
    xp = W.hidden_states(sh, B, P, wl.seed, 0, "bf16")
    xs = [W.hidden_states(sh, B, 1, wl.seed, 1 + t, "bf16") for t in range(T)]
    wd = dev(w)
    kc, vc = _zeros_cache(B, nkv, cap, hd), _zeros_cache(B, nkv, cap, hd)
    q = torch.empty((B, nh, P, hd), dtype=BF, device="cuda")
    o_p = torch.empty((B, P, nh, hd), dtype=BF, device="cuda")
    posp = np.broadcast_to(np.arange(P, dtype=np.int32), (B, P)).copy()
    gqa.qkv_rope_project(dev(xp), wd, dev_i32(posp), nh, nkv, hd, sh.rope_theta, q, kc, vc)
    gqa.gqa_attn_prefill(q, kc, vc, dev_i32(np.full(B, P)), True, o_p)
    ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap), dtype=torch.uint8, device="cuda")
    check = {0, 1, 2, 100, 511, 1022, 1023}
    outs = {}
    qt = torch.empty((B, nh, 1, hd), dtype=BF, device="cuda")
    xs_d = [dev(x) for x in xs]
    for t in range(T):
        pos_t = torch.full((B, 1), P + t, dtype=torch.int32, device="cuda")
        gqa.qkv_rope_project(xs_d[t], wd, pos_t, nh, nkv, hd, sh.rope_theta, qt, kc, vc)
        ot = torch.empty((B, nh, hd), dtype=BF, device="cuda")
        gqa.gqa_attn_decode(qt.view(B, nh, hd), kc, vc, torch.full((B,), P + t + 1, dtype=torch.int32,
                                                                     device="cuda"), ot, ws)
        if t in check:
            outs[t] = ot
    torch.cuda.synchronize()

    # oracle: all tokens projected at once (step inputs are independent draws)
    x_all = np.concatenate([xp.f64] + [x.f64 for x in xs], axis=1)
    pos_all = np.broadcast_to(np.arange(P + T), (B, P + T))
    z = np.zeros((B, nkv, cap, hd))
    q_r, kc_r, vc_r = ref.qkv_rope_project(x_all, w.f64, pos_all, nh, nkv, hd, sh.rope_theta, z, z)
    # attention reads the bf16 q/K/V that the projection stored
    rq, rk, rv = ref.round_bf16(q_r), ref.round_bf16(kc_r), ref.round_bf16(vc_r)
    o_pr = ref.prefill_attention(rq[:, :, :P], rk, rv, np.full(B, P), True)
    gate(host(o_p), o_pr, "bf16", "prompt prefill")
    for t, ot in outs.items():
        d_r = ref.decode_attention(rq[:, :, P + t], rk, rv, np.full(B, P + t + 1))
        gate(host(ot), d_r, "bf16", f"decode step {t}")
    gate(host(kc), kc_r, "bf16", "final K cache")
    gate(host(vc), vc_r, "bf16", "final V cache")


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("nkv", W.LONG_PREFILL.extra["n_kv_heads_cases"])
def test_long_prefill_outliers(nkv, causal):
    wl = W.LONG_PREFILL
    B, S = wl.batch_seq[0]
    nh, hd = wl.shape.n_heads, wl.shape.head_dim
    q, k, v = W.outlier_qkv(B, S, nh, nkv, hd, wl.seed + nkv)
    out = torch.empty((B, S, nh, hd), dtype=BF, device="cuda")
    gqa.gqa_attn_prefill(dev(q), dev(k), dev(v), dev_i32(np.full(B, S)), causal, out)
    got = host(out)
    r = np.random.default_rng(2)
    rows = [(int(r.integers(B)), h, int(r.integers(S))) for h in range(nh) for _ in range(8)]
    rows += [(0, 0, 0), (1, nh - 1, S - 1), (0, 3, 127), (1, 5, 128), (0, 7, 4095)]
    want = ref.prefill_attention(q.f64, k.f64, v.f64, np.full(B, S), causal, rows=rows)
    # V's outlier channels (x20) give the output channels of every query head
    # reading that KV head a 20x scale (attention is linear in V)
    vscale = np.ones(nkv * hd)
    vscale[W.outlier_channels(nkv * hd, 0.001, wl.seed + nkv, 2)] = 20.0
    vscale = vscale.reshape(nkv, hd)
    g = nh // nkv
    gate(np.stack([got[b, s, h] for b, h, s in rows]), want, "bf16", f"long prefill nkv={nkv} causal={causal}",
         col_scale=np.stack([vscale[h // g] for _, h, _ in rows]))
    assert np.all(np.isfinite(got))
