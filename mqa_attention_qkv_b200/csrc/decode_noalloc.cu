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
// device current) on the first call made on that device.
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

// Device address of g_decode_scratch on the current device.  In host code the
// array's name is only a host-side stand-in: a kernel given it would fault (or
// silently use the wrong memory), so the real address is looked up here.
void* scratch_ptr() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  ScratchSlot& s = g_slot[dev];
  std::call_once(s.once, [&] {
    s.status = cudaGetSymbolAddress(&s.ptr, g_decode_scratch);
    // the split counters at the front must start at zero; every call leaves them so
    if (s.status == cudaSuccess) s.status = cudaMemset(s.ptr, 0, kNoAllocScratchBytes);
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
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || n_heads <= 0 || n_kv_heads <= 0 || cache_cap <= 0) return GQA_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads != 0) return GQA_ERR_INVALID_ARG;
  if (kv_split < 0 || (kv_split > 0 && kv_split % 64)) return GQA_ERR_INVALID_ARG;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return GQA_ERR_UNSUPPORTED_SHAPE;
  if ((long long)B * n_kv_heads * cache_cap * head_dim > (1ll << 40) || B > 65535 || n_kv_heads > 65535 ||
      (long long)B * n_kv_heads * cache_cap >= (1ll << 31))   // 32-bit cache row coordinates
    return GQA_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return GQA_OK;
  if (!q || !k_cache || !v_cache || !kv_lens || !out) return GQA_ERR_INVALID_ARG;
  const auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(q) || !a16(k_cache) || !a16(v_cache) || !a16(out) || (reinterpret_cast<uintptr_t>(kv_lens) & 3u))
    return GQA_ERR_MISALIGNED;
  // The problem's partials must fit the fixed scratch; larger problems are
  // rejected (a larger kv_split needs fewer partials).
  const size_t need = gqa_attn_decode_workspace_size(B, n_heads, n_kv_heads, head_dim, cache_cap, kv_split);
  if (need == 0 || need > kNoAllocScratchBytes) return GQA_ERR_WORKSPACE_TOO_SMALL;
  int* err = nullptr;
  const int st = gqa::device_check(&err);
  if (st != GQA_OK) return st;
  void* ws = scratch_ptr();
  if (!ws) return GQA_ERR_NO_DEVICE;

  // The scratch starts with the per-(sequence, KV head) split counters, which
  // must be zero: the set-up above zeroes the array once and every call leaves
  // the counters at zero again.  The partials need no clearing (each one the
  // merge reads is written by the same call first).  Calls that overlap on the
  // GPU (other streams) share the array and race; order them on one stream or
  // with events.
  const gqa::DecodeParams p = gqa::decode_params(q, k_cache, v_cache, kv_lens, B, n_heads, n_kv_heads, head_dim,
                                                 cache_cap, kv_split, out, ws, err);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  gqa::count_launches(gqa::launch_decode(p, dtype == GQA_BF16, s, &e));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_LAUNCH_FAILED;
  }
  return GQA_OK;
}

}  // extern "C"
