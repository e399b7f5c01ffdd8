// gqa_attn_decode_noalloc: the split-KV decode with its scratch in a fixed,
// file-scope device array instead of a caller-provided workspace.
//
// Who needs it: callers that cannot call cudaMalloc (or ask an allocator for
// device memory) at the point where they run decode - for example a serving
// loop whose device memory is entirely pre-reserved by another allocator, a
// plugin handed only the tensors of the op by its host framework with no
// allocator interface, or a latency-critical path where an allocation (which
// may synchronise the device) is not allowed.  They still pass every input
// and output; only the scratch lives inside the library.
//
// The scratch array is kNoAllocScratchBytes (64 MiB) of device memory that
// every GPU which loads this library holds until the process exits.  Its
// device address is looked up once per device (cudaGetSymbolAddress with that
// device current) on the first call made on that device; each call clears the
// split counters at its front with an asynchronous memset on its own stream.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/gqa.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 64ull << 20;

// The decode partials (per sequence, query head and key split: o[hd], m, l).
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

struct ScratchSlot {
  std::once_flag once;
  void* ptr = nullptr;
  cudaError_t status = cudaSuccess;
};
ScratchSlot g_slot[kMaxDevices];

// Device address of g_decode_scratch on the current device, looked up once
// per device with that device current.  In host code the array's name is only
// a host-side stand-in: a kernel given it would fault (or silently use the
// wrong memory), so the real address is taken from the runtime.
void* scratch_ptr() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  ScratchSlot& s = g_slot[dev];
  std::call_once(s.once, [&] {
    s.status = cudaGetSymbolAddress(&s.ptr, g_decode_scratch);
    if (s.status != cudaSuccess) {
      s.ptr = nullptr;
      cudaGetLastError();
    }
  });
  return s.status == cudaSuccess ? s.ptr : nullptr;
}

}  // namespace

extern "C" {

int gqa_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* kv_lens, int B, int n_heads, int n_kv_heads, int head_dim,
                            int cache_cap, int kv_split, void* out, int dtype, void* stream) {
  // the same validation as gqa_attn_decode, minus the workspace arguments
  if (const int v = gqa::decode_check_args(q, k_cache, v_cache, kv_lens, B, n_heads, n_kv_heads, head_dim,
                                           cache_cap, kv_split, out, dtype);
      v != GQA_OK || B == 0)
    return v;
  // The problem's counters and partials must fit the fixed scratch; larger
  // problems are rejected (a larger kv_split needs fewer partials).
  const size_t need = gqa_attn_decode_workspace_size(B, n_heads, n_kv_heads, head_dim, cache_cap, kv_split);
  if (need == 0 || need > kNoAllocScratchBytes) return GQA_ERR_WORKSPACE_TOO_SMALL;
  int* err = nullptr;
  const int st = gqa::device_check(&err);
  if (st != GQA_OK) return st;
  void* ws = scratch_ptr();
  if (!ws) return GQA_ERR_NO_DEVICE;

  // The scratch starts with the per-(sequence, KV head, head group) split
  // counters, which must start at zero.  The array keeps whatever the last
  // call left, so they are cleared here, on the caller's stream, ahead of the
  // decode kernel (stream order makes the clear finish first whatever kind of
  // stream the caller uses).  The partials need no clearing: every partial
  // the merge reads is written by the same call first.  Calls that overlap on
  // the GPU (other streams) share the array and race; order them on one
  // stream or with events.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t counter_bytes =
      gqa::decode_counter_bytes(B, n_kv_heads, gqa::decode_n_hgrp(n_heads, n_kv_heads));
  if (cudaMemsetAsync(ws, 0, counter_bytes, s) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_LAUNCH_FAILED;
  }
  const gqa::DecodeParams p = gqa::decode_params(q, k_cache, v_cache, kv_lens, B, n_heads, n_kv_heads, head_dim,
                                                 cache_cap, kv_split, out, ws, err);
  cudaError_t e;
  gqa::count_launches(gqa::launch_decode(p, dtype == GQA_BF16, s, &e));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_LAUNCH_FAILED;
  }
  return GQA_OK;
}

}  // extern "C"
