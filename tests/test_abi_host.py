"""C-ABI checks that need no GPU: the library loads, exports every function
the header declares, and rejects bad arguments on the host before any device
work (so these calls never touch the fake pointers they are given)."""
import ctypes
import os
import re

import pytest

import mqa_attention_qkv_b200 as gqa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa.h")

# 16-byte aligned, never dereferenced: every call below fails validation first.
P = 0x100000
MIS = P + 8


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?(?:int|size_t|uint64_t|char\s*\*|void)\s*\*?\s*(\w+)\s*\(",
                                 src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert set(names) == set(gqa.EXPORTED_SYMBOLS), names
    L = ctypes.CDLL(gqa.library_path())
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8):
        s = gqa.gqa_status_string(code)
        assert s and s != "unknown status"
    assert gqa.gqa_status_string(12345) == "unknown status"


def _qkv(**kw):
    a = dict(x=P, w=P, pos=P, B=2, S=4, hidden=64, nh=4, nkv=2, hd=64, theta=1e4,
             q=P, k=P, v=P, cap=16, dtype=1, stream=None)
    a.update(kw)
    return gqa.lib().qkv_rope_project(a["x"], a["w"], a["pos"], a["B"], a["S"], a["hidden"], a["nh"],
                                      a["nkv"], a["hd"], a["theta"], a["q"], a["k"], a["v"], a["cap"],
                                      a["dtype"], a["stream"])


def _prefill(**kw):
    a = dict(q=P, k=P, v=P, qpos=None, lens=P, B=2, S=4, nh=4, nkv=2, hd=64, cap=16, causal=1,
             out=P, dtype=1, stream=None)
    a.update(kw)
    return gqa.lib().gqa_attn_prefill(a["q"], a["k"], a["v"], a["qpos"], a["lens"], a["B"], a["S"],
                                      a["nh"], a["nkv"], a["hd"], a["cap"], a["causal"], a["out"],
                                      a["dtype"], a["stream"])


def _decode(**kw):
    a = dict(q=P, k=P, v=P, lens=P, B=2, nh=4, nkv=2, hd=64, cap=16, split=0, out=P, ws=P,
             ws_bytes=1 << 30, dtype=1, stream=None)
    a.update(kw)
    return gqa.lib().gqa_attn_decode(a["q"], a["k"], a["v"], a["lens"], a["B"], a["nh"], a["nkv"],
                                     a["hd"], a["cap"], a["split"], a["out"], a["ws"], a["ws_bytes"],
                                     a["dtype"], a["stream"])


INVALID, MISALIGNED, DTYPE, ARCH, WS, LAUNCH, SHAPE, NODEV = -1, -2, -3, -4, -5, -6, -7, -8


@pytest.mark.parametrize("kw,code", [
    (dict(x=None), INVALID), (dict(w=None), INVALID), (dict(pos=None), INVALID),
    (dict(q=None), INVALID), (dict(k=None), INVALID), (dict(v=None), INVALID),
    (dict(nh=6, nkv=4), INVALID), (dict(nkv=0), INVALID), (dict(B=-1), INVALID),
    (dict(S=-3), INVALID), (dict(hidden=0), INVALID), (dict(cap=0), INVALID),
    (dict(theta=0.0), INVALID), (dict(hd=96), SHAPE), (dict(hd=256), SHAPE), (dict(dtype=2), DTYPE),
    (dict(x=MIS), MISALIGNED), (dict(k=MIS), MISALIGNED), (dict(pos=P + 2), MISALIGNED),
])
def test_qkv_rejects(kw, code):
    assert _qkv(**kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(lens=None), INVALID), (dict(out=None), INVALID),
    (dict(nh=3, nkv=2), INVALID), (dict(cap=0), INVALID), (dict(hd=16), SHAPE),
    (dict(dtype=-1), DTYPE), (dict(out=MIS), MISALIGNED), (dict(qpos=P + 1), MISALIGNED),
    (dict(B=2, nkv=2, cap=1 << 29), SHAPE),             # 2^31 cache rows
    (dict(B=1, nh=4, nkv=2, S=1 << 29), SHAPE),         # 2^31 query rows
])
def test_prefill_rejects(kw, code):
    assert _prefill(**kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(ws=None), INVALID), (dict(lens=None), INVALID), (dict(split=100), INVALID),
    (dict(split=-64), INVALID), (dict(nh=4, nkv=3), INVALID), (dict(hd=48), SHAPE),
    (dict(ws_bytes=16), WS), (dict(ws=MIS), MISALIGNED), (dict(dtype=7), DTYPE),
    (dict(B=2, nkv=2, nh=4, cap=1 << 29, split=1 << 21), SHAPE),   # 2^31 cache rows
])
def test_decode_rejects(kw, code):
    assert _decode(**kw) == code


def _decode_noalloc(**kw):
    a = dict(q=P, k=P, v=P, lens=P, B=2, nh=4, nkv=2, hd=64, cap=16, split=0, out=P, dtype=1, stream=None)
    a.update(kw)
    return gqa.lib().gqa_attn_decode_noalloc(a["q"], a["k"], a["v"], a["lens"], a["B"], a["nh"], a["nkv"],
                                             a["hd"], a["cap"], a["split"], a["out"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw", [
    dict(q=None), dict(k=None), dict(v=None), dict(lens=None), dict(out=None), dict(split=100),
    dict(split=-64), dict(nh=4, nkv=3), dict(nkv=0), dict(B=-1), dict(cap=0), dict(hd=48),
    dict(q=MIS), dict(out=MIS), dict(lens=P + 2), dict(dtype=7),
    dict(cap=64 * 600, split=64),                                    # 600 splits > 512
    dict(B=2, nkv=2, nh=4, cap=1 << 29, split=1 << 21),              # 2^31 cache rows
])
def test_noalloc_decode_validates_like_decode(kw):
    """Both decode entry points run the same argument checks."""
    want = _decode(**kw)
    assert want < 0
    assert _decode_noalloc(**kw) == want


def _meanpool(**kw):
    a = dict(w=P, hidden=64, nh=8, nkv=2, hd=64, out=P + (1 << 24), dtype=1, stream=None)
    a.update(kw)
    return gqa.lib().gqa_meanpool_kv_heads(a["w"], a["hidden"], a["nh"], a["nkv"], a["hd"], a["out"], a["dtype"],
                                           a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(w=None), INVALID), (dict(out=None), INVALID), (dict(nh=6, nkv=4), INVALID), (dict(nkv=0), INVALID),
    (dict(hidden=0), INVALID), (dict(hd=-64), INVALID), (dict(hidden=60), SHAPE), (dict(hidden=6, dtype=0), SHAPE),
    (dict(dtype=5), DTYPE), (dict(w=MIS), MISALIGNED), (dict(out=P + (1 << 24) + 4), MISALIGNED),
    (dict(out=P + 4096), INVALID),   # output overlaps the input
])
def test_meanpool_rejects(kw, code):
    assert _meanpool(**kw) == code


def _paged(**kw):
    a = dict(q=P, k=P, v=P, table=P, lens=P, B=2, nh=8, nkv=2, hd=128, ps=64, maxp=4, nump=8, split=0, out=P,
             ws=P, ws_bytes=1 << 30, dtype=1, stream=None)
    a.update(kw)
    return gqa.lib().gqa_attn_decode_paged(a["q"], a["k"], a["v"], a["table"], a["lens"], a["B"], a["nh"],
                                           a["nkv"], a["hd"], a["ps"], a["maxp"], a["nump"], a["split"], a["out"],
                                           a["ws"], a["ws_bytes"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(table=None), INVALID), (dict(lens=None), INVALID), (dict(k=None), INVALID), (dict(ws=None), INVALID),
    (dict(ps=0), INVALID), (dict(ps=96), INVALID), (dict(maxp=0), INVALID), (dict(nump=0), INVALID),
    (dict(nh=6, nkv=4), INVALID), (dict(split=100), INVALID), (dict(split=-64), INVALID),
    (dict(hd=32), SHAPE), (dict(hd=96), SHAPE), (dict(dtype=0), DTYPE),
    (dict(ps=1 << 20, maxp=1 << 12), SHAPE),          # 2^32 keys a sequence
    (dict(ps=1 << 16, nump=1 << 15), SHAPE),          # 2^32 cache rows
    (dict(ws_bytes=16), WS), (dict(table=P + 2), MISALIGNED), (dict(v=MIS), MISALIGNED),
])
def test_paged_decode_rejects(kw, code):
    assert _paged(**kw) == code


def _varlen(**kw):
    a = dict(q=P, k=P, v=P, cq=P, ck=P, B=2, tq=300, tk=300, maxq=200, nh=8, nkv=2, hd=64, causal=1, out=P,
             dtype=1, stream=None)
    a.update(kw)
    return gqa.lib().gqa_attn_prefill_varlen(a["q"], a["k"], a["v"], a["cq"], a["ck"], a["B"], a["tq"], a["tk"],
                                             a["maxq"], a["nh"], a["nkv"], a["hd"], a["causal"], a["out"],
                                             a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(cq=None), INVALID), (dict(ck=None), INVALID), (dict(k=None), INVALID), (dict(out=None), INVALID),
    (dict(B=-1), INVALID), (dict(tq=-1), INVALID), (dict(tk=-5), INVALID), (dict(maxq=-1), INVALID),
    (dict(nh=6, nkv=4), INVALID), (dict(nkv=0), INVALID), (dict(hd=32), SHAPE), (dict(hd=96), SHAPE),
    (dict(dtype=0), DTYPE), (dict(cq=P + 2), MISALIGNED), (dict(q=MIS), MISALIGNED),
    (dict(tq=1 << 30, nh=2048, nkv=2048), SHAPE),              # 2^47 query elements
    (dict(B=60000, maxq=1 << 20, nh=64, nkv=8), SHAPE),        # grid of 2^31 tiles or more
])
def test_varlen_prefill_rejects(kw, code):
    assert _varlen(**kw) == code


def test_empty_inputs_are_noops():
    # B == 0 or S == 0 returns OK without launching (pointers may then be NULL)
    assert _qkv(B=0, x=None, w=None, pos=None, q=None, k=None, v=None) == 0
    assert _qkv(S=0) == 0
    assert _prefill(B=0, q=None) == 0
    assert _prefill(S=0) == 0
    assert _decode(B=0, q=None, ws=None) == 0
    assert _paged(B=0, q=None, table=None, ws=None) == 0
    assert _varlen(B=0, q=None, cq=None) == 0
    assert _varlen(tq=0) == 0
    assert _varlen(maxq=0) == 0


def test_workspace_size_query():
    f = gqa.gqa_attn_decode_workspace_size
    # split counters (B * nkv * ceil(g / 16) words, rounded up to 256 bytes)
    # then B * nh * ceil(cap / split) * (hd + 4) floats
    assert f(2, 4, 2, 64, 1000, 64) == 256 + 2 * 4 * 16 * 68 * 4
    assert f(64, 32, 8, 128, 8192, 512) == 2048 + 64 * 32 * 16 * 132 * 4
    assert f(64, 32, 1, 128, 8192, 512) == 512 + 64 * 32 * 16 * 132 * 4    # g = 32: 2 head groups
    assert f(8, 48, 1, 128, 1040, 64) == 256 + 8 * 48 * 17 * 132 * 4       # g = 48: 3 head groups
    assert f(2, 4, 2, 64, 1000, 0) > 0
    assert f(2, 4, 2, 64, 1000, 100) == 0      # split not a multiple of 64
    assert f(2, 4, 3, 64, 1000, 64) == 0       # nh % nkv
    assert f(2, 4, 2, 80, 1000, 64) == 0       # head_dim


def test_valid_call_without_gpu_reports_no_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; this case is for GPU-less hosts")
    assert _qkv() in (NODEV, ARCH)
    assert _prefill() in (NODEV, ARCH)
    assert _decode() in (NODEV, ARCH)
    assert _meanpool() in (NODEV, ARCH)
    assert _paged() in (NODEV, ARCH)
    assert _varlen() in (NODEV, ARCH)
    assert _varlen(tk=0) in (NODEV, ARCH)      # no keys at all: zero rows


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    """No fallback: with the shared library absent every call raises."""
    monkeypatch.setattr(gqa, "_LIB", None)
    monkeypatch.setattr(gqa, "library_path", lambda: str(tmp_path / "libgqa_b200.so"))
    with pytest.raises(ImportError):
        gqa.lib()
    with pytest.raises(ImportError):
        gqa.gqa_attn_decode_workspace_size(1, 8, 1, 128, 64)
    with pytest.raises(ImportError):
        gqa.gqa_launch_count()


def test_binding_rejects_host_tensors():
    """Tensors must live on the GPU: host tensors are refused before any
    library call."""
    import torch
    q = torch.zeros(2, 8, 64, dtype=torch.bfloat16)
    kc = torch.zeros(2, 2, 64, 64, dtype=torch.bfloat16)
    lens = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        gqa.gqa_attn_decode(q, kc, kc, lens, q.clone(), torch.zeros(1024, dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        gqa.gqa_attn_decode_paged(q, kc, kc, torch.zeros(2, 1, dtype=torch.int32), lens, q.clone(),
                                  torch.zeros(1024, dtype=torch.uint8))


def test_skip_tile_knob_validates_on_the_host():
    assert gqa.lib().gqa_debug_skip_next_kv_tile(-2) == INVALID
    assert gqa.lib().gqa_debug_skip_next_kv_tile(-1) == 0     # disarm


def test_injected_launch_failures_are_reported_then_clear():
    """Host-side fault injection: after validation, the next n compute calls
    report GQA_ERR_LAUNCH_FAILED without launching; invalid calls are still
    refused first and do not use an injection."""
    assert gqa.lib().gqa_debug_inject_launch_failures(-1) == INVALID
    n0 = gqa.gqa_launch_count()
    gqa.gqa_debug_inject_launch_failures(3)
    try:
        assert _decode(dtype=7) == DTYPE
        assert _decode() == LAUNCH
        assert _qkv() == LAUNCH
        assert _meanpool() == LAUNCH
        if not _gpu_present():
            assert _decode() in (NODEV, ARCH)     # the injections are used up
    finally:
        gqa.gqa_debug_inject_launch_failures(0)
    assert gqa.gqa_launch_count() == n0            # nothing was launched
    with pytest.raises(gqa.GQAError) as e:
        gqa._check("gqa_attn_decode", LAUNCH)
    assert e.value.status == LAUNCH and "launch failed" in str(e.value)


def _gpu_present():
    import torch
    return torch.cuda.is_available()


def test_binding_argument_lists_match_the_header():
    """Every declared function is bound with as many arguments as the header
    gives it (catches drift between include/gqa.h and the ctypes binding)."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decl = re.compile(r"^\s*(?:const\s+)?(?:int|size_t|uint64_t|char\s*\*|void)\s*\*?\s*(\w+)\s*\(([^)]*)\)\s*;",
                      re.M)
    L = gqa.lib()
    seen = 0
    for name, params in decl.findall(src):
        params = params.strip()
        n = 0 if params in ("", "void") else len(params.split(","))
        argtypes = getattr(L, name).argtypes
        assert argtypes is not None and len(argtypes) == n, (name, n, argtypes)
        seen += 1
    assert seen == len(gqa.EXPORTED_SYMBOLS)
