// C ABI of libgqa_b200: host-side argument validation, kernel selection and
// launch on the caller's stream.  No allocation, no synchronisation, no
// printing (gqa_device_error, a debugging aid, is the one synchronising call).
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "../../include/gqa.h"
#include "kernels.h"

namespace {

// Device error block, one per device in the library's static device memory:
// word 0 the GQA_DEVERR_* bits, words 2-3 a wait-limit override in ns (0 =
// the default; set only by gqa_debug_set_wait_limit_ns).
__device__ __align__(16) int g_device_error[4];

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  std::once_flag once;
  int cc_major = 0, cc_minor = 0, num_sms = 0;
  int* err = nullptr;
  cudaError_t status = cudaSuccess;
};
DeviceInfo g_dev[kMaxDevices];
std::atomic<unsigned long long> g_launches{0};

// Per-device facts, queried once with that device current.
const DeviceInfo* device_info(int* status) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    *status = GQA_ERR_NO_DEVICE;
    return nullptr;
  }
  DeviceInfo& d = g_dev[dev];
  std::call_once(d.once, [&] {
    cudaError_t e = cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_device_error);
    d.status = e;
    if (e != cudaSuccess) cudaGetLastError();
  });
  if (d.status != cudaSuccess) {
    *status = GQA_ERR_NO_DEVICE;
    return nullptr;
  }
  if (d.cc_major != 10 || d.cc_minor != 0) {
    *status = GQA_ERR_UNSUPPORTED_ARCH;
    return nullptr;
  }
  *status = GQA_OK;
  return &d;
}

// Launch failures injected by gqa_debug_inject_launch_failures: the next n
// compute calls that pass validation report GQA_ERR_LAUNCH_FAILED without
// launching anything.
std::atomic<int> g_inject_failures{0};
// gqa_debug_skip_next_kv_tile: K tile + 1 that the next head-dim-64 prefill's
// first CTA does not load (0 = none); taken by that call.
std::atomic<int> g_skip_kv_tile{0};

bool take_injected_failure() {
  int n = g_inject_failures.load(std::memory_order_relaxed);
  while (n > 0)
    if (g_inject_failures.compare_exchange_weak(n, n - 1, std::memory_order_relaxed)) return true;
  return false;
}

// Device facts for a compute call (an injected failure is reported here,
// after argument validation and before any launch).
const DeviceInfo* compute_device(int* status) {
  if (take_injected_failure()) {
    *status = GQA_ERR_LAUNCH_FAILED;
    return nullptr;
  }
  return device_info(status);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool hd_ok(int hd) { return hd == 32 || hd == 64 || hd == 128; }

int launch_status(cudaError_t e, int n_launched = 1) {
  g_launches.fetch_add((unsigned long long)n_launched, std::memory_order_relaxed);
  if (e == cudaSuccess) return GQA_OK;
  cudaGetLastError();
  return GQA_ERR_LAUNCH_FAILED;
}

// Keys per decode split when the caller leaves it to the library: about two
// work units (sequence x KV head x group of 16 query heads x split) per SM of
// a B200 (148 SMs) for a full cache, at least 128 keys (2 tiles) and at most
// 2048, a multiple of 64, and never more than kMaxSplits splits.  (Eight
// units per SM, tried for ragged MQA batches, measured slower on B200.)
constexpr long long kUnitsWanted = 2 * 148;
using gqa::kMaxSplits;
int auto_split(int B, int nkv, int n_hgrp, int cap) {
  const long long groups = (long long)B * nkv * n_hgrp;
  long long s = (groups * cap + kUnitsWanted - 1) / kUnitsWanted;
  s = (s + 63) / 64 * 64;
  if (s < 128) s = 128;
  if (s > 2048) s = 2048;
  const long long min_s = ((cap + kMaxSplits - 1) / kMaxSplits + 63) / 64 * 64;
  if (s < min_s) s = min_s;
  return (int)s;
}

constexpr long long kMaxElems = 1ll << 40;
// Rows of the tensor-map views ([B*nkv*cap, hd] caches, [B*nh*S, hd] queries)
// are addressed with 32-bit coordinates and int row arithmetic.
constexpr long long kMaxRows = 1ll << 31;

}  // namespace

namespace gqa {

int device_check(int** err) {
  int st;
  const DeviceInfo* d = compute_device(&st);
  if (d && err) *err = d->err;
  return st;
}

void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

int decode_split_len(int B, int nh, int nkv, int cache_cap, int kv_split) {
  return kv_split ? kv_split : auto_split(B, nkv, decode_n_hgrp(nh, nkv), cache_cap);
}

int decode_check_args(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_lens, int B,
                      int nh, int nkv, int hd, int cap, int kv_split, const void* out, int dtype) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || nh <= 0 || nkv <= 0 || cap <= 0) return GQA_ERR_INVALID_ARG;
  if (nh % nkv != 0) return GQA_ERR_INVALID_ARG;
  if (kv_split < 0 || (kv_split > 0 && kv_split % 64)) return GQA_ERR_INVALID_ARG;
  if (kv_split > 0 && (cap + kv_split - 1) / kv_split > kMaxSplits) return GQA_ERR_INVALID_ARG;
  if (!hd_ok(hd)) return GQA_ERR_UNSUPPORTED_SHAPE;
  if ((long long)B * nkv * cap * hd > kMaxElems || B > 65535 || nkv > 65535 || (long long)B * nkv * cap >= kMaxRows)
    return GQA_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return GQA_OK;
  if (!q || !k_cache || !v_cache || !kv_lens || !out) return GQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned4(kv_lens))
    return GQA_ERR_MISALIGNED;
  return GQA_OK;
}

DecodeParams decode_params(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_lens,
                           int B, int nh, int nkv, int hd, int cap, int kv_split, void* out, void* workspace,
                           int* err) {
  const int split = decode_split_len(B, nh, nkv, cap, kv_split);
  const int n_hgrp = decode_n_hgrp(nh, nkv);
  unsigned* counters = static_cast<unsigned*>(workspace);
  float* partials = reinterpret_cast<float*>(static_cast<char*>(workspace) + decode_counter_bytes(B, nkv, n_hgrp));
  return DecodeParams{q, k_cache, v_cache, kv_lens, B, nh, nkv, hd, cap, split, (cap + split - 1) / split,
                      partials, out, err, counters, n_hgrp, kv_split == 0, 0, nullptr, 0, 0, 0};
}

}  // namespace gqa

extern "C" {

const char* gqa_status_string(int status) {
  switch (status) {
    case GQA_OK: return "ok";
    case GQA_ERR_INVALID_ARG: return "invalid argument";
    case GQA_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case GQA_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype";
    case GQA_ERR_UNSUPPORTED_ARCH: return "device is not compute capability 10.0 (sm_100a)";
    case GQA_ERR_WORKSPACE_TOO_SMALL: return "decode workspace too small";
    case GQA_ERR_LAUNCH_FAILED: return "kernel launch failed";
    case GQA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (head_dim must be 32, 64 or 128)";
    case GQA_ERR_NO_DEVICE: return "no usable CUDA device";
    default: return "unknown status";
  }
}

int gqa_device_error(int* bits) {
  if (!bits) return GQA_ERR_INVALID_ARG;
  int st;
  const DeviceInfo* d = device_info(&st);
  if (!d) return st;
  int v = 0;
  const int zero = 0;
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpy(&v, d->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(d->err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_LAUNCH_FAILED;
  }
  *bits = v;
  return GQA_OK;
}

int qkv_rope_project(const void* x, const void* w_qkv, const int32_t* positions,
                     int B, int S, int hidden, int n_heads, int n_kv_heads, int head_dim,
                     float rope_theta, void* q_out, void* k_cache, void* v_cache,
                     int cache_cap, int dtype, void* stream) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || S < 0 || hidden <= 0 || n_heads <= 0 || n_kv_heads <= 0 || cache_cap <= 0)
    return GQA_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads != 0) return GQA_ERR_INVALID_ARG;
  if (!(rope_theta > 0.f)) return GQA_ERR_INVALID_ARG;
  if (!hd_ok(head_dim)) return GQA_ERR_UNSUPPORTED_SHAPE;
  if ((long long)B * S * hidden > kMaxElems || (long long)B * S >= (1ll << 31) ||
      (long long)(n_heads + 2 * n_kv_heads) * head_dim * hidden > kMaxElems)
    return GQA_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || S == 0) return GQA_OK;
  if (!x || !w_qkv || !positions || !q_out || !k_cache || !v_cache) return GQA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q_out) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned4(positions))
    return GQA_ERR_MISALIGNED;
  int st;
  const DeviceInfo* d = compute_device(&st);
  if (!d) return st;

  gqa::QkvParams p{x, w_qkv, positions, B, S, hidden, n_heads, n_kv_heads, head_dim, cache_cap,
                   (double)rope_theta, q_out, k_cache, v_cache, d->err};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Tensor-core path: bf16 with 16-byte-aligned rows (TMA row stride).
  if (dtype == GQA_BF16 && hidden % 8 == 0) {
    // a few tokens: W-streaming kernel spread over every SM; else 128-token tiles
    if ((long long)B * S <= 64) return launch_status(gqa::launch_qkv_smallm(p, d->num_sms, s));
    return launch_status(gqa::launch_qkv_tc(p, d->num_sms, s));
  }
  return launch_status(gqa::launch_qkv_simt(p, dtype == GQA_BF16, s));
}

int gqa_attn_prefill(const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* q_positions, const int32_t* kv_lens,
                     int B, int S, int n_heads, int n_kv_heads, int head_dim,
                     int cache_cap, int causal, void* out, int dtype, void* stream) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || S < 0 || n_heads <= 0 || n_kv_heads <= 0 || cache_cap <= 0) return GQA_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads != 0) return GQA_ERR_INVALID_ARG;
  if (!hd_ok(head_dim)) return GQA_ERR_UNSUPPORTED_SHAPE;
  if ((long long)B * n_kv_heads * cache_cap * head_dim > kMaxElems ||
      (long long)B * n_heads * S * head_dim > kMaxElems || B > 65535 || n_heads > 65535 ||
      (long long)B * n_kv_heads * cache_cap >= kMaxRows || (long long)B * n_heads * S >= kMaxRows)
    return GQA_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || S == 0) return GQA_OK;
  if (!q || !k_cache || !v_cache || !kv_lens || !out) return GQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned4(kv_lens) || (q_positions && !aligned4(q_positions)))
    return GQA_ERR_MISALIGNED;
  int st;
  const DeviceInfo* d = compute_device(&st);
  if (!d) return st;

  gqa::PrefillParams p{q, k_cache, v_cache, q_positions, kv_lens, B, S, n_heads, n_kv_heads,
                       head_dim, cache_cap, causal ? 1 : 0, out, d->err};
  if (dtype == GQA_BF16 && head_dim == 64) p.dbg_skip_tile1 = g_skip_kv_tile.exchange(0);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // head_dim 64: two CTAs per SM (measured fastest there); 128: two query tiles per CTA
  if (dtype == GQA_BF16 && head_dim == 64) return launch_status(gqa::launch_prefill_pair(p, s));
  if (dtype == GQA_BF16 && head_dim == 128) return launch_status(gqa::launch_prefill_fa(p, s));
  return launch_status(gqa::launch_prefill_simt(p, dtype == GQA_BF16, s));
}

int gqa_attn_prefill_varlen(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                            const int32_t* cu_seqlens_k, int B, int total_q, int total_k, int max_seqlen_q,
                            int n_heads, int n_kv_heads, int head_dim, int causal, void* out, int dtype,
                            void* stream) {
  if (dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || n_heads <= 0 || n_kv_heads <= 0)
    return GQA_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads != 0) return GQA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return GQA_ERR_UNSUPPORTED_SHAPE;
  if ((long long)total_q * n_heads * head_dim > kMaxElems || (long long)total_k * n_kv_heads * head_dim > kMaxElems ||
      B > 65535 || n_heads > 65535 || (long long)B * n_heads * ((max_seqlen_q + 127) / 128) >= kMaxRows)
    return GQA_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || total_q == 0 || max_seqlen_q == 0) return GQA_OK;
  if (!q || !k || !v || !cu_seqlens_q || !cu_seqlens_k || !out) return GQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned4(cu_seqlens_q) ||
      !aligned4(cu_seqlens_k))
    return GQA_ERR_MISALIGNED;
  int st;
  const DeviceInfo* d = compute_device(&st);
  if (!d) return st;

  gqa::PrefillParams p{q, k, v, nullptr, nullptr, B, max_seqlen_q, n_heads, n_kv_heads, head_dim, total_k,
                       causal ? 1 : 0, out, d->err, cu_seqlens_q, cu_seqlens_k, total_q};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (head_dim == 64) return launch_status(gqa::launch_prefill_pair(p, s));
  return launch_status(gqa::launch_prefill_fa(p, s));
}

size_t gqa_attn_decode_workspace_size(int B, int n_heads, int n_kv_heads, int head_dim,
                                      int cache_cap, int kv_split) {
  if (B < 0 || n_heads <= 0 || n_kv_heads <= 0 || cache_cap <= 0 || n_heads % n_kv_heads) return 0;
  if (!hd_ok(head_dim)) return 0;
  if (kv_split < 0 || (kv_split > 0 && kv_split % 64)) return 0;
  const int split = gqa::decode_split_len(B, n_heads, n_kv_heads, cache_cap, kv_split);
  const size_t n_split = (size_t)(cache_cap + split - 1) / split;
  if (n_split > (size_t)kMaxSplits) return 0;
  size_t partials = (size_t)B * n_heads * n_split * (head_dim + gqa::kWsPad) * sizeof(float);
  // the keys-as-rows decode (bf16) takes its own partial slots
  if (gqa::decode_hn_ok(B, n_heads, n_kv_heads, head_dim, cache_cap, kv_split == 0)) {
    const size_t hn = gqa::decode_hn_partial_bytes(B, n_heads, n_kv_heads);
    if (hn > partials) partials = hn;
  }
  return gqa::decode_counter_bytes(B, n_kv_heads, gqa::decode_n_hgrp(n_heads, n_kv_heads)) + partials;
}

int gqa_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* kv_lens, int B, int n_heads, int n_kv_heads, int head_dim,
                    int cache_cap, int kv_split, void* out, void* workspace,
                    size_t workspace_bytes, int dtype, void* stream) {
  if (const int v = gqa::decode_check_args(q, k_cache, v_cache, kv_lens, B, n_heads, n_kv_heads, head_dim,
                                           cache_cap, kv_split, out, dtype);
      v != GQA_OK || B == 0)
    return v;
  if (!workspace) return GQA_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return GQA_ERR_MISALIGNED;
  const size_t need = gqa_attn_decode_workspace_size(B, n_heads, n_kv_heads, head_dim, cache_cap, kv_split);
  if (workspace_bytes < need) return GQA_ERR_WORKSPACE_TOO_SMALL;
  int st;
  const DeviceInfo* d = compute_device(&st);
  if (!d) return st;

  const gqa::DecodeParams p = gqa::decode_params(q, k_cache, v_cache, kv_lens, B, n_heads, n_kv_heads, head_dim,
                                                 cache_cap, kv_split, out, workspace, d->err);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  const int n = gqa::launch_decode(p, dtype == GQA_BF16, s, &e);
  return launch_status(e, n);
}

int gqa_attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                          const int32_t* block_table, const int32_t* kv_lens, int B, int n_heads,
                          int n_kv_heads, int head_dim, int page_size, int max_pages, int num_pages,
                          int kv_split, void* out, void* workspace, size_t workspace_bytes, int dtype,
                          void* stream) {
  if (dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
  if (B < 0 || n_heads <= 0 || n_kv_heads <= 0 || page_size <= 0 || max_pages <= 0 || num_pages <= 0)
    return GQA_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads != 0 || page_size % 64) return GQA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return GQA_ERR_UNSUPPORTED_SHAPE;
  const long long cap = (long long)max_pages * page_size;
  // every cache row index (page, KV head, row) stays a 32-bit int
  if (cap >= kMaxRows || (long long)num_pages * n_kv_heads * page_size >= kMaxRows ||
      (long long)B * max_pages >= (1ll << 31) || B > 65535 || n_kv_heads > 65535)
    return GQA_ERR_UNSUPPORTED_SHAPE;
  if (kv_split < 0 || (kv_split > 0 && kv_split % 64)) return GQA_ERR_INVALID_ARG;
  if (kv_split > 0 && (cap + kv_split - 1) / kv_split > kMaxSplits) return GQA_ERR_INVALID_ARG;
  if (B == 0) return GQA_OK;
  if (!q || !k_pages || !v_pages || !block_table || !kv_lens || !out || !workspace) return GQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(out) ||
      !aligned16(workspace) || !aligned4(kv_lens) || !aligned4(block_table))
    return GQA_ERR_MISALIGNED;
  const size_t need = gqa_attn_decode_workspace_size(B, n_heads, n_kv_heads, head_dim, (int)cap, kv_split);
  if (need == 0) return GQA_ERR_UNSUPPORTED_SHAPE;
  if (workspace_bytes < need) return GQA_ERR_WORKSPACE_TOO_SMALL;
  int st;
  const DeviceInfo* d = compute_device(&st);
  if (!d) return st;

  gqa::DecodeParams p = gqa::decode_params(q, k_pages, v_pages, kv_lens, B, n_heads, n_kv_heads, head_dim,
                                           (int)cap, kv_split, out, workspace, d->err);
  p.block_table = block_table;
  p.page_size = page_size;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  const int n = gqa::launch_decode(p, true, s, &e);
  return launch_status(e, n);
}

int gqa_o_proj_residual(const void* attn, const void* w_o, const void* residual, int T, int n_heads,
                        int head_dim, int hidden, void* out, int dtype, void* stream) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
  if (T < 0 || n_heads <= 0 || hidden <= 0) return GQA_ERR_INVALID_ARG;
  if (!hd_ok(head_dim)) return GQA_ERR_UNSUPPORTED_SHAPE;
  const long long K = (long long)n_heads * head_dim;
  if ((long long)T * K > kMaxElems || (long long)T * hidden > kMaxElems || K * hidden > kMaxElems ||
      K >= kMaxRows || (long long)T >= kMaxRows)
    return GQA_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return GQA_OK;
  if (!attn || !w_o || !out) return GQA_ERR_INVALID_ARG;
  if (!aligned16(attn) || !aligned16(w_o) || !aligned16(out) || (residual && !aligned16(residual)))
    return GQA_ERR_MISALIGNED;
  // out may be the residual itself (in place); no other overlap is allowed
  const size_t es = dtype == GQA_BF16 ? 2 : 4;
  const char* ob = static_cast<const char*>(out);
  const size_t ob_n = (size_t)T * hidden * es;
  auto overlaps = [&](const void* q, size_t n) {
    const char* qb = static_cast<const char*>(q);
    return qb < ob + ob_n && ob < qb + n;
  };
  if (overlaps(attn, (size_t)T * K * es) || overlaps(w_o, (size_t)K * hidden * es) ||
      (residual && residual != out && overlaps(residual, ob_n)))
    return GQA_ERR_INVALID_ARG;
  int st;
  const DeviceInfo* d = compute_device(&st);
  if (!d) return st;

  const gqa::OprojParams p{attn, w_o, residual, out, T, (int)K, hidden, d->err};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == GQA_BF16 && hidden % 8 == 0) {
    if (T <= 64) {
      // W_o-bound: the few-token projection's streaming kernel where its
      // shape rules hold, else the cluster-split tensor-core kernel
      if (gqa::oproj_stream_fits(p)) return launch_status(gqa::launch_oproj_stream(p, d->num_sms, s));
      return launch_status(gqa::launch_oproj_smallt(p, d->num_sms, s));
    }
    return launch_status(gqa::launch_oproj_tc(p, d->num_sms, s));
  }
  return launch_status(gqa::launch_oproj_simt(p, dtype == GQA_BF16, s));
}

uint64_t gqa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int gqa_fp8_quantize_qkv(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_lens, int B,
                         int S, int n_heads, int n_kv_heads, int head_dim, int cache_cap, const int8_t* signs,
                         void* q8, void* k8, void* v8t, float* amax, void* stream) {
  if (B < 0 || S < 0 || n_heads <= 0 || n_kv_heads <= 0 || cache_cap <= 0) return GQA_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads != 0) return GQA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return GQA_ERR_UNSUPPORTED_SHAPE;
  if (cache_cap % 16 != 0) return GQA_ERR_UNSUPPORTED_SHAPE;   // 16-byte rows of the transposed V
  if ((long long)B * n_kv_heads * cache_cap * head_dim > kMaxElems || (long long)B * n_heads * S * head_dim > kMaxElems ||
      (long long)B * n_kv_heads * cache_cap >= kMaxRows || (long long)B * n_heads * S >= kMaxRows)
    return GQA_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return GQA_OK;
  if (!q || !k_cache || !v_cache || !kv_lens || !q8 || !k8 || !v8t || !amax) return GQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q8) || !aligned16(k8) ||
      !aligned16(v8t) || !aligned4(kv_lens) || !aligned4(amax))
    return GQA_ERR_MISALIGNED;
  gqa::Fp8QuantParams p{q, k_cache, v_cache, kv_lens, B, S, n_heads, n_kv_heads, head_dim, cache_cap,
                        signs != nullptr, {0u, 0u, 0u, 0u}, q8, k8, v8t, amax, nullptr};
  if (signs) {
    for (int c = 0; c < head_dim; ++c) {
      if (signs[c] != 1 && signs[c] != -1) return GQA_ERR_INVALID_ARG;
      if (signs[c] < 0) p.signs[c >> 5] |= 1u << (c & 31);
    }
  }
  int st;
  const DeviceInfo* d = compute_device(&st);
  if (!d) return st;
  p.err = d->err;
  return launch_status(gqa::launch_fp8_quantize(p, d->num_sms, static_cast<cudaStream_t>(stream)), 3);
}

int gqa_attn_prefill_fp8(const void* q8, const void* k8, const void* v8t, const float* amax, const int32_t* kv_lens,
                         int B, int S, int n_heads, int n_kv_heads, int head_dim, int cache_cap, int causal, void* out,
                         void* stream) {
  if (B < 0 || S < 0 || n_heads <= 0 || n_kv_heads <= 0 || cache_cap <= 0) return GQA_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads != 0) return GQA_ERR_INVALID_ARG;
  if (head_dim != 128 || cache_cap % 16 != 0) return GQA_ERR_UNSUPPORTED_SHAPE;
  if ((long long)B * n_kv_heads * cache_cap * head_dim > kMaxElems || (long long)B * n_heads * S * head_dim > kMaxElems ||
      B > 65535 || n_heads > 65535 || (long long)B * n_kv_heads * cache_cap >= kMaxRows ||
      (long long)B * n_heads * S >= kMaxRows)
    return GQA_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || S == 0) return GQA_OK;
  if (!q8 || !k8 || !v8t || !amax || !kv_lens || !out) return GQA_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8t) || !aligned16(out) || !aligned4(amax) || !aligned4(kv_lens))
    return GQA_ERR_MISALIGNED;
  int st;
  const DeviceInfo* d = compute_device(&st);
  if (!d) return st;
  const gqa::Fp8AttnParams p{q8, k8, v8t, amax, kv_lens, B, S, n_heads, n_kv_heads, head_dim, cache_cap,
                             causal ? 1 : 0, out, d->err};
  return launch_status(gqa::launch_prefill_fp8(p, static_cast<cudaStream_t>(stream)));
}

int gqa_debug_set_wait_limit_ns(uint64_t ns) {
  int st;
  const DeviceInfo* d = device_info(&st);
  if (!d) return st;
  if (cudaMemcpy(d->err + 2, &ns, sizeof(ns), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_LAUNCH_FAILED;
  }
  return GQA_OK;
}

int gqa_debug_exp2_poly(const float* x, int n, float* poly, float* ref, void* stream) {
  if (n < 0) return GQA_ERR_INVALID_ARG;
  if (n == 0) return GQA_OK;
  if (!x || !poly || !ref) return GQA_ERR_INVALID_ARG;
  if (!aligned4(x) || !aligned4(poly) || !aligned4(ref)) return GQA_ERR_MISALIGNED;
  int st;
  const DeviceInfo* d = device_info(&st);
  if (!d) return st;
  return launch_status(gqa::launch_exp2_check(x, n, poly, ref, static_cast<cudaStream_t>(stream)));
}

int gqa_debug_skip_next_kv_tile(int tile) {
  if (tile < -1) return GQA_ERR_INVALID_ARG;
  g_skip_kv_tile.store(tile + 1);
  return GQA_OK;
}

int gqa_debug_inject_launch_failures(int n) {
  if (n < 0) return GQA_ERR_INVALID_ARG;
  g_inject_failures.store(n, std::memory_order_relaxed);
  return GQA_OK;
}

}  // extern "C"
