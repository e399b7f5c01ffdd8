"""gqa_attn_decode_noalloc: decode for callers that cannot allocate device
memory where they run it (a serving loop whose device memory another
allocator has fully reserved, a plugin that gets only the op's tensors, a
path on which a possibly synchronising allocation is not allowed).

Its split-KV scratch is a fixed static array inside the library, so the
check is that it returns what the workspace-taking gqa_attn_decode returns,
within the bf16 tolerance of the parity tests, on two calls in a row (the
second call finds the first call's partials still in the shared array), and
that a problem too large for the array is refused.

This file is collected last so that a run stopping at its first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

import mqa_attention_qkv_b200 as gqa
import workloads as W
from tests._helpers import dev, dev_i32, gate, host

pytestmark = pytest.mark.gpu


def _problem(seed, B, nh, nkv, hd, cap, lens):
    q = W.normal_tensor((B, nh, hd), seed, 0, "bf16")
    kc = W.decode_cache(seed, 1, B, nkv, cap, hd, lens)
    vc = W.decode_cache(seed, 2, B, nkv, cap, hd, lens)
    return dev(q), dev(kc), dev(vc), dev_i32(lens)


def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    cases = [
        # seed, B, n_heads, n_kv_heads, head_dim, cache_cap, kv_lens, kv_split
        (31, 8, 32, 8, 128, 2048, np.array([2048, 1, 777, 1500, 64, 65, 1999, 300], dtype=np.int32), 0),
        (32, 5, 48, 1, 64, 700, np.array([700, 13, 640, 129, 400], dtype=np.int32), 64),
    ]
    for seed, B, nh, nkv, hd, cap, lens, split in cases:
        q, kc, vc, ln = _problem(seed, B, nh, nkv, hd, cap, lens)
        ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap, split),
                         dtype=torch.uint8, device="cuda")
        want = torch.empty((B, nh, hd), dtype=torch.bfloat16, device="cuda")
        got = torch.full((B, nh, hd), float("nan"), dtype=torch.bfloat16, device="cuda")
        gqa.gqa_attn_decode(q, kc, vc, ln, want, ws, kv_split=split)
        gqa.gqa_attn_decode_noalloc(q, kc, vc, ln, got, kv_split=split)
        torch.cuda.synchronize()
        gate(host(got), host(want), "bf16", f"no-alloc decode, seed {seed}")


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
