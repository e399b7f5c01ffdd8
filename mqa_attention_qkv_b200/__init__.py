"""Python binding of libgqa_b200 (fused-QKV projection + grouped-query
attention for B200 / sm_100a).

Argument marshalling only: shapes are read from the torch tensors, pointers
and sizes are passed to the C ABI declared in ``include/gqa.h``, and every step
of the computation runs in the library's CUDA kernels.  PyTorch provides the
device memory and the stream.  There is no other code path: if the shared
library is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "GQA_F32", "GQA_BF16", "GQAError", "library_path", "lib",
    "qkv_rope_project", "gqa_attn_prefill", "gqa_attn_decode",
    "gqa_attn_decode_workspace_size", "gqa_status_string", "gqa_device_error",
    "gqa_launch_count", "gqa_attn_decode_noalloc", "gqa_meanpool_kv_heads", "gqa_attn_decode_paged",
    "gqa_attn_prefill_varlen", "gqa_debug_inject_launch_failures", "gqa_o_proj_residual",
    "gqa_debug_set_wait_limit_ns", "gqa_debug_skip_next_kv_tile", "gqa_fp8_quantize_qkv",
    "gqa_attn_prefill_fp8", "gqa_debug_exp2_poly", "EXPORTED_SYMBOLS",
]

GQA_F32 = 0
GQA_BF16 = 1

EXPORTED_SYMBOLS = (
    "qkv_rope_project", "gqa_attn_prefill", "gqa_attn_decode",
    "gqa_attn_decode_workspace_size", "gqa_status_string", "gqa_device_error",
    "gqa_launch_count", "gqa_attn_decode_noalloc", "gqa_meanpool_kv_heads", "gqa_attn_decode_paged",
    "gqa_attn_prefill_varlen", "gqa_debug_inject_launch_failures", "gqa_o_proj_residual",
    "gqa_debug_set_wait_limit_ns", "gqa_debug_skip_next_kv_tile", "gqa_fp8_quantize_qkv",
    "gqa_attn_prefill_fp8", "gqa_debug_exp2_poly",
)

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


class GQAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {gqa_status_string(status)} (status {status})")
        self.status = status


def library_path() -> str:
    return os.path.join(_HERE, "libgqa_b200.so")


def lib() -> ctypes.CDLL:
    """The loaded shared library (loaded on first use; raises if absent)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run `python -m mqa_attention_qkv_b200.build`")
    L = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.qkv_rope_project.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, ctypes.c_float,
                                   vp, vp, vp, i32, i32, vp]
    L.qkv_rope_project.restype = i32
    L.gqa_attn_prefill.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, i32, vp]
    L.gqa_attn_prefill.restype = i32
    L.gqa_attn_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
    L.gqa_attn_decode_workspace_size.restype = sz
    L.gqa_attn_decode.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, sz, i32, vp]
    L.gqa_attn_decode.restype = i32
    L.gqa_status_string.argtypes = [i32]
    L.gqa_status_string.restype = ctypes.c_char_p
    L.gqa_device_error.argtypes = [ctypes.POINTER(ctypes.c_int)]
    L.gqa_device_error.restype = i32
    L.gqa_launch_count.argtypes = []
    L.gqa_launch_count.restype = ctypes.c_uint64
    L.gqa_attn_decode_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, i32, vp]
    L.gqa_attn_decode_noalloc.restype = i32
    L.gqa_meanpool_kv_heads.argtypes = [vp, i32, i32, i32, i32, vp, i32, vp]
    L.gqa_meanpool_kv_heads.restype = i32
    L.gqa_attn_decode_paged.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp, sz,
                                        i32, vp]
    L.gqa_attn_decode_paged.restype = i32
    L.gqa_attn_prefill_varlen.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, i32, vp]
    L.gqa_attn_prefill_varlen.restype = i32
    L.gqa_o_proj_residual.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, i32, vp]
    L.gqa_o_proj_residual.restype = i32
    L.gqa_fp8_quantize_qkv.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    L.gqa_fp8_quantize_qkv.restype = i32
    L.gqa_attn_prefill_fp8.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp]
    L.gqa_attn_prefill_fp8.restype = i32
    L.gqa_debug_exp2_poly.argtypes = [vp, i32, vp, vp, vp]
    L.gqa_debug_exp2_poly.restype = i32
    L.gqa_debug_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.gqa_debug_set_wait_limit_ns.restype = i32
    L.gqa_debug_skip_next_kv_tile.argtypes = [i32]
    L.gqa_debug_skip_next_kv_tile.restype = i32
    L.gqa_debug_inject_launch_failures.argtypes = [i32]
    L.gqa_debug_inject_launch_failures.restype = i32
    _LIB = L
    return L


def gqa_status_string(status: int) -> str:
    return lib().gqa_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != 0:
        raise GQAError(fn, status)


# --------------------------------------------------------------------------
# tensor marshalling helpers
# --------------------------------------------------------------------------
def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return GQA_BF16
    if t.dtype == torch.float32:
        return GQA_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16 or torch.float32")


def _ptr(t, dtype=None, shape=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


# --------------------------------------------------------------------------
# the three calls
# --------------------------------------------------------------------------
def qkv_rope_project(x, w_qkv, positions, n_heads: int, n_kv_heads: int, head_dim: int,
                     rope_theta: float, q_out, k_cache, v_cache, stream=None) -> None:
    """x [B,S,hidden], w_qkv [(nh+2nkv)*hd, hidden], positions [B,S] int32 ->
    q_out [B,nh,S,hd]; k_cache/v_cache [B,nkv,cap,hd] written at slot=position."""
    import torch
    B, S, hidden = x.shape
    dt = x.dtype
    cap = k_cache.shape[2]
    n_qkv = (n_heads + 2 * n_kv_heads) * head_dim
    args = (
        _ptr(x, dt, name="x"), _ptr(w_qkv, dt, (n_qkv, hidden), "w_qkv"),
        _ptr(positions, torch.int32, (B, S), "positions"),
        B, S, hidden, n_heads, n_kv_heads, head_dim, float(rope_theta),
        _ptr(q_out, dt, (B, n_heads, S, head_dim), "q_out"),
        _ptr(k_cache, dt, (B, n_kv_heads, cap, head_dim), "k_cache"),
        _ptr(v_cache, dt, (B, n_kv_heads, cap, head_dim), "v_cache"),
        cap, _dtype_code(x), _stream(stream),
    )
    _check("qkv_rope_project", lib().qkv_rope_project(*args))


def gqa_attn_prefill(q, k_cache, v_cache, kv_lens, causal: bool, out, q_positions=None,
                     stream=None) -> None:
    """q [B,nh,S,hd], caches [B,nkv,cap,hd], kv_lens [B] int32 -> out [B,S,nh,hd]."""
    import torch
    B, nh, S, hd = q.shape
    nkv, cap = k_cache.shape[1], k_cache.shape[2]
    dt = q.dtype
    args = (
        _ptr(q, dt, name="q"), _ptr(k_cache, dt, (B, nkv, cap, hd), "k_cache"),
        _ptr(v_cache, dt, (B, nkv, cap, hd), "v_cache"),
        _ptr(q_positions, torch.int32, (B, S), "q_positions"),
        _ptr(kv_lens, torch.int32, (B,), "kv_lens"),
        B, S, nh, nkv, hd, cap, 1 if causal else 0,
        _ptr(out, dt, (B, S, nh, hd), "out"), _dtype_code(q), _stream(stream),
    )
    _check("gqa_attn_prefill", lib().gqa_attn_prefill(*args))


def gqa_attn_decode_workspace_size(B: int, n_heads: int, n_kv_heads: int, head_dim: int,
                                   cache_cap: int, kv_split: int = 0) -> int:
    return int(lib().gqa_attn_decode_workspace_size(B, n_heads, n_kv_heads, head_dim, cache_cap, kv_split))


def gqa_attn_decode(q, k_cache, v_cache, kv_lens, out, workspace, kv_split: int = 0,
                    stream=None) -> None:
    """q [B,nh,hd], caches [B,nkv,cap,hd], kv_lens [B] int32 -> out [B,nh,hd].
    ``workspace`` is a CUDA tensor of at least gqa_attn_decode_workspace_size bytes."""
    import torch
    B, nh, hd = q.shape
    nkv, cap = k_cache.shape[1], k_cache.shape[2]
    dt = q.dtype
    ws_bytes = workspace.numel() * workspace.element_size()
    args = (
        _ptr(q, dt, name="q"), _ptr(k_cache, dt, (B, nkv, cap, hd), "k_cache"),
        _ptr(v_cache, dt, (B, nkv, cap, hd), "v_cache"),
        _ptr(kv_lens, torch.int32, (B,), "kv_lens"),
        B, nh, nkv, hd, cap, int(kv_split),
        _ptr(out, dt, (B, nh, hd), "out"), _ptr(workspace, name="workspace"), ws_bytes,
        _dtype_code(q), _stream(stream),
    )
    _check("gqa_attn_decode", lib().gqa_attn_decode(*args))


def gqa_attn_prefill_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, causal: bool, out,
                            stream=None) -> None:
    """Packed variable-length prefill: q [total_q,nh,hd], k/v [total_k,nkv,hd]
    bf16, cu_seqlens_q/k [B+1] int32 -> out [total_q,nh,hd] (include/gqa.h)."""
    import torch
    total_q, nh, hd = q.shape
    total_k, nkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.shape[0] - 1
    dt = q.dtype
    args = (
        _ptr(q, dt, name="q"), _ptr(k, dt, (total_k, nkv, hd), "k"), _ptr(v, dt, (total_k, nkv, hd), "v"),
        _ptr(cu_seqlens_q, torch.int32, (B + 1,), "cu_seqlens_q"),
        _ptr(cu_seqlens_k, torch.int32, (B + 1,), "cu_seqlens_k"),
        B, total_q, total_k, int(max_seqlen_q), nh, nkv, hd, int(bool(causal)),
        _ptr(out, dt, (total_q, nh, hd), "out"), _dtype_code(q), _stream(stream),
    )
    _check("gqa_attn_prefill_varlen", lib().gqa_attn_prefill_varlen(*args))


def gqa_attn_decode_paged(q, k_pages, v_pages, block_table, kv_lens, out, workspace, kv_split: int = 0,
                          stream=None) -> None:
    """q [B,nh,hd] bf16, pages [num_pages,nkv,page_size,hd] bf16, block_table
    [B,max_pages] int32, kv_lens [B] int32 -> out [B,nh,hd].  ``workspace`` as
    for gqa_attn_decode with cache_cap = max_pages * page_size."""
    import torch
    B, nh, hd = q.shape
    num_pages, nkv, page_size = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    max_pages = block_table.shape[1]
    dt = q.dtype
    ws_bytes = workspace.numel() * workspace.element_size()
    args = (
        _ptr(q, dt, name="q"), _ptr(k_pages, dt, (num_pages, nkv, page_size, hd), "k_pages"),
        _ptr(v_pages, dt, (num_pages, nkv, page_size, hd), "v_pages"),
        _ptr(block_table, torch.int32, (B, max_pages), "block_table"),
        _ptr(kv_lens, torch.int32, (B,), "kv_lens"),
        B, nh, nkv, hd, page_size, max_pages, num_pages, int(kv_split),
        _ptr(out, dt, (B, nh, hd), "out"), _ptr(workspace, name="workspace"), ws_bytes,
        _dtype_code(q), _stream(stream),
    )
    _check("gqa_attn_decode_paged", lib().gqa_attn_decode_paged(*args))


def gqa_o_proj_residual(attn, w_o, out, residual=None, stream=None) -> None:
    """Output projection + residual: attn [..., nh, hd] (the heads of each
    token in order), w_o [hidden, nh*hd], residual None or [..., hidden] ->
    out [..., hidden] = attn . w_o^T + residual.  ``out`` may be ``residual``
    (in place)."""
    *lead, nh, hd = attn.shape
    T = 1
    for d in lead:
        T *= int(d)
    hidden = w_o.shape[0]
    dt = attn.dtype
    oshape = (*lead, hidden)
    args = (
        _ptr(attn, dt, name="attn"), _ptr(w_o, dt, (hidden, nh * hd), "w_o"),
        _ptr(residual, dt, oshape, "residual"), T, nh, hd, hidden,
        _ptr(out, dt, oshape, "out"), _dtype_code(attn), _stream(stream),
    )
    _check("gqa_o_proj_residual", lib().gqa_o_proj_residual(*args))


def gqa_fp8_quantize_qkv(q, k_cache, v_cache, kv_lens, q8, k8, v8t, amax, signs=None, stream=None) -> None:
    """FP8 inputs for gqa_attn_prefill_fp8: q [B,nh,S,hd], caches [B,nkv,cap,hd]
    bf16 -> q8 [B,nh,S,hd], k8 [B,nkv,cap,hd], v8t [B,nkv,hd,cap] (uint8
    tensors holding e4m3 codes) and amax [3] float32; ``signs`` (hd values
    +-1, a host sequence) selects the random-sign Hadamard rotation of q and
    k, None for none."""
    import torch
    B, nh, S, hd = q.shape
    nkv, cap = k_cache.shape[1], k_cache.shape[2]
    sg = None
    if signs is not None:
        sg = (ctypes.c_int8 * hd)(*[int(v) for v in signs])
    args = (
        _ptr(q, torch.bfloat16, name="q"), _ptr(k_cache, torch.bfloat16, (B, nkv, cap, hd), "k_cache"),
        _ptr(v_cache, torch.bfloat16, (B, nkv, cap, hd), "v_cache"), _ptr(kv_lens, torch.int32, (B,), "kv_lens"),
        B, S, nh, nkv, hd, cap, ctypes.cast(sg, ctypes.c_void_p) if sg is not None else None,
        _ptr(q8, torch.uint8, (B, nh, S, hd), "q8"), _ptr(k8, torch.uint8, (B, nkv, cap, hd), "k8"),
        _ptr(v8t, torch.uint8, (B, nkv, hd, cap), "v8t"), _ptr(amax, torch.float32, (3,), "amax"), _stream(stream),
    )
    _check("gqa_fp8_quantize_qkv", lib().gqa_fp8_quantize_qkv(*args))


def gqa_attn_prefill_fp8(q8, k8, v8t, amax, kv_lens, causal: bool, out, stream=None) -> None:
    """FP8 prefill: the tensors of gqa_fp8_quantize_qkv -> out [B,S,nh,hd] bf16."""
    import torch
    B, nh, S, hd = q8.shape
    nkv, cap = k8.shape[1], k8.shape[2]
    args = (
        _ptr(q8, torch.uint8, name="q8"), _ptr(k8, torch.uint8, (B, nkv, cap, hd), "k8"),
        _ptr(v8t, torch.uint8, (B, nkv, hd, cap), "v8t"), _ptr(amax, torch.float32, (3,), "amax"),
        _ptr(kv_lens, torch.int32, (B,), "kv_lens"), B, S, nh, nkv, hd, cap, 1 if causal else 0,
        _ptr(out, torch.bfloat16, (B, S, nh, hd), "out"), _stream(stream),
    )
    _check("gqa_attn_prefill_fp8", lib().gqa_attn_prefill_fp8(*args))


def gqa_device_error() -> int:
    """Read and clear the device error word (synchronises the device)."""
    v = ctypes.c_int(0)
    _check("gqa_device_error", lib().gqa_device_error(ctypes.byref(v)))
    return v.value


def gqa_debug_inject_launch_failures(n: int) -> None:
    """Testing aid: the next ``n`` compute calls fail as a failed launch would
    (GQAError with status GQA_ERR_LAUNCH_FAILED), launching nothing."""
    _check("gqa_debug_inject_launch_failures", lib().gqa_debug_inject_launch_failures(int(n)))


def gqa_debug_set_wait_limit_ns(ns: int) -> None:
    """Testing aid: pipeline waits give up after ``ns`` nanoseconds (0 = the
    default 2 s) on the current device, from the next launch on."""
    _check("gqa_debug_set_wait_limit_ns", lib().gqa_debug_set_wait_limit_ns(int(ns)))


def gqa_debug_skip_next_kv_tile(tile: int) -> None:
    """Testing aid: the next head_dim-64 bf16 prefill leaves key tile ``tile``
    unloaded in its first CTA, so that the waits on it run out (-1 disarms)."""
    _check("gqa_debug_skip_next_kv_tile", lib().gqa_debug_skip_next_kv_tile(int(tile)))


def gqa_debug_exp2_poly(x, poly, ref, stream=None) -> None:
    """Testing aid: the softmax's polynomial 2^x (poly) and CUDA's exp2f (ref)
    for the float32 CUDA tensor x."""
    import torch
    n = x.numel()
    args = (_ptr(x, torch.float32, name="x"), n, _ptr(poly, torch.float32, (n,), "poly"),
            _ptr(ref, torch.float32, (n,), "ref"), _stream(stream))
    _check("gqa_debug_exp2_poly", lib().gqa_debug_exp2_poly(*args))


def gqa_launch_count() -> int:
    """Kernels launched by the library so far in this process (host counter)."""
    return int(lib().gqa_launch_count())


def gqa_attn_decode_noalloc(q, k_cache, v_cache, kv_lens, out, kv_split: int = 0, stream=None) -> None:
    """gqa_attn_decode for callers that cannot allocate device memory: the
    split-KV scratch is a fixed 64 MiB static array inside the library (see
    include/gqa.h).  Same shapes and results as gqa_attn_decode."""
    import torch
    B, nh, hd = q.shape
    nkv, cap = k_cache.shape[1], k_cache.shape[2]
    dt = q.dtype
    args = (
        _ptr(q, dt, name="q"), _ptr(k_cache, dt, (B, nkv, cap, hd), "k_cache"),
        _ptr(v_cache, dt, (B, nkv, cap, hd), "v_cache"),
        _ptr(kv_lens, torch.int32, (B,), "kv_lens"),
        B, nh, nkv, hd, cap, int(kv_split),
        _ptr(out, dt, (B, nh, hd), "out"), _dtype_code(q), _stream(stream),
    )
    _check("gqa_attn_decode_noalloc", lib().gqa_attn_decode_noalloc(*args))


def gqa_meanpool_kv_heads(w_qkv_mha, n_heads: int, n_kv_heads: int, head_dim: int, w_qkv_gqa,
                          stream=None) -> None:
    """MHA -> GQA weight transform: w_qkv_mha [3*nh*hd, hidden] -> w_qkv_gqa
    [(nh + 2*nkv)*hd, hidden], each group's key/value projections mean-pooled
    (include/gqa.h)."""
    dt = w_qkv_mha.dtype
    hidden = w_qkv_mha.shape[1]
    args = (
        _ptr(w_qkv_mha, dt, (3 * n_heads * head_dim, hidden), "w_qkv_mha"), hidden, n_heads, n_kv_heads, head_dim,
        _ptr(w_qkv_gqa, dt, ((n_heads + 2 * n_kv_heads) * head_dim, hidden), "w_qkv_gqa"),
        _dtype_code(w_qkv_mha), _stream(stream),
    )
    _check("gqa_meanpool_kv_heads", lib().gqa_meanpool_kv_heads(*args))

