"""gqa_attn_decode_noalloc: decode for callers that cannot allocate device
memory where they run it (a serving loop whose device memory another
allocator has fully reserved, a plugin that gets only the op's tensors, a
path on which a possibly synchronising allocation is not allowed).

Its split-KV scratch is a fixed static array inside the library.  The
parametrised cases pass an explicit kv_split, so the decode merges its
splits through that array (split counters plus partials) rather than inside
a thread-block cluster; one more case leaves the split to the library on a
problem that takes the keys-as-rows decode, whose pieces merge through the
same array.  Two calls in a row with different inputs must each give what the
workspace-taking gqa_attn_decode gives and what the float64 oracle gives,
within the bf16 gate of the parity tests: the second call starts from the
counters and partials the first one left in the shared array.  A fresh
process whose first call runs on a non-blocking stream checks the per-call
counter clear, and a problem too large for the array is refused.

This file is collected last so that a run stopping at its first failure has
already run every other test.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import mqa_attention_qkv_b200 as gqa
import workloads as W
from oracle import gqa_ref as ref
from tests._helpers import dev, dev_i32, gate, host

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# seed, B, n_heads, n_kv_heads, head_dim, cache_cap, kv_lens, kv_split, dtype
CASES = [
    (31, 8, 32, 8, 128, 2048, [2048, 1, 777, 1500, 64, 65, 1999, 300], 256, "bf16"),
    (32, 5, 48, 1, 64, 700, [700, 13, 640, 129, 400], 64, "bf16"),
    (33, 3, 8, 2, 32, 300, [300, 1, 190], 64, "f32"),
]


def _problem(seed, B, nh, nkv, hd, cap, lens, dtype):
    q = W.normal_tensor((B, nh, hd), seed, 0, dtype)
    kc = W.decode_cache(seed, 1, B, nkv, cap, hd, lens, dtype)
    vc = W.decode_cache(seed, 2, B, nkv, cap, hd, lens, dtype)
    want = ref.decode_attention(q.f64, kc.f64, vc.f64, lens)
    return (dev(q), dev(kc), dev(vc), dev_i32(lens)), want


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"seed{c[0]}-{c[8]}-hd{c[4]}-split{c[7]}")
def test_noalloc_decode_matches_workspace_decode_on_two_calls(case):
    seed, B, nh, nkv, hd, cap, lens, split, dt = case
    lens = np.array(lens, dtype=np.int32)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap, split), dtype=torch.uint8,
                     device="cuda")
    # two calls in a row on different inputs (the second reversed lengths and
    # another seed), each checked against gqa_attn_decode and the oracle
    for call, (s, ln) in enumerate(((seed, lens), (seed + 100, lens[::-1].copy()))):
        (q, kc, vc, lnd), want = _problem(s, B, nh, nkv, hd, cap, ln, dt)
        base = torch.empty((B, nh, hd), dtype=tdt, device="cuda")
        got = torch.full((B, nh, hd), float("nan"), dtype=tdt, device="cuda")
        gqa.gqa_attn_decode(q, kc, vc, lnd, base, ws, kv_split=split)
        gqa.gqa_attn_decode_noalloc(q, kc, vc, lnd, got, kv_split=split)
        torch.cuda.synchronize()
        gate(host(got), host(base), dt, f"no-alloc vs workspace decode, call {call}")
        gate(host(got), want, dt, f"no-alloc decode vs oracle, call {call}")


def test_noalloc_keys_as_rows_decode_on_two_calls():
    """The library's own split on a problem that takes the keys-as-rows
    decode (B 16, 32 heads on one KV head, hd 128, a 20000-key cache): its
    split counters and per-piece partials live in the static array; two calls
    in a row with different lengths each match gqa_attn_decode and the
    oracle."""
    B, nh, nkv, hd, cap = 16, 32, 1, 128, 20000
    rng = np.random.default_rng(41)
    ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap, 0), dtype=torch.uint8, device="cuda")
    for call in range(2):
        lens = np.array([cap, 1, 0, 8191] + list(rng.integers(1, cap + 1, size=B - 4)), dtype=np.int32)
        (q, kc, vc, lnd), want = _problem(50 + call, B, nh, nkv, hd, cap, lens, "bf16")
        base = torch.empty((B, nh, hd), dtype=torch.bfloat16, device="cuda")
        got = torch.full((B, nh, hd), float("nan"), dtype=torch.bfloat16, device="cuda")
        gqa.gqa_attn_decode(q, kc, vc, lnd, base, ws)
        gqa.gqa_attn_decode_noalloc(q, kc, vc, lnd, got)
        torch.cuda.synchronize()
        g = host(got)
        assert np.all(g[2] == 0)
        keep = lens > 0
        gate(g[keep], host(base)[keep], "bf16", f"no-alloc vs workspace keys-as-rows decode, call {call}")
        gate(g[keep], want[keep], "bf16", f"no-alloc keys-as-rows decode vs oracle, call {call}")


_FRESH = r"""
import sys
sys.path.insert(0, sys.argv[1])
import numpy as np, torch
import mqa_attention_qkv_b200 as gqa
import workloads as W
from oracle import gqa_ref as ref
from tests._helpers import dev, dev_i32, gate, host
torch.cuda.set_device(0)
B, nh, nkv, hd, cap, split = 6, 32, 4, 128, 1024, 128
lens = np.array([1024, 3, 500, 129, 900, 64], dtype=np.int32)
q = W.normal_tensor((B, nh, hd), 41, 0, "bf16")
kc = W.decode_cache(41, 1, B, nkv, cap, hd, lens)
vc = W.decode_cache(41, 2, B, nkv, cap, hd, lens)
want = ref.decode_attention(q.f64, kc.f64, vc.f64, lens)
side = torch.cuda.Stream()          # a non-blocking stream: no implicit order with the legacy stream
with torch.cuda.stream(side):
    qd, kd, vd, ld = dev(q), dev(kc), dev(vc), dev_i32(lens)
    out = torch.full((B, nh, hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    gqa.gqa_attn_decode_noalloc(qd, kd, vd, ld, out, kv_split=split)   # the first call of this process
side.synchronize()
gate(host(out), want, "bf16", "first no-alloc call on a side stream")
print("fresh ok")
"""


def test_noalloc_first_call_on_a_side_stream_in_a_fresh_process():
    r = subprocess.run([sys.executable, "-c", _FRESH, ROOT], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "fresh ok" in r.stdout, r.stdout + r.stderr


def test_noalloc_decode_refuses_problems_larger_than_its_scratch():
    B, nh, nkv, hd, cap, split = 64, 32, 1, 128, 8192, 64
    need = gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap, split)
    assert need > 64 << 20
    q = torch.zeros((B, nh, hd), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((B, nkv, cap, hd), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ln = torch.full((B,), cap, dtype=torch.int32, device="cuda")
    out = torch.zeros((B, nh, hd), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gqa.GQAError) as e:
        gqa.gqa_attn_decode_noalloc(q, kc, vc, ln, out, kv_split=split)
    assert e.value.status == -5
