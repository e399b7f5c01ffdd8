// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <utility>

namespace gqa {

struct QkvParams {
  const void* x;          // [T, hidden]      T = B*S
  const void* w;          // [N, hidden]      N = (nh + 2 nkv) * hd
  const int32_t* pos;     // [T]
  int B, S, hidden, nh, nkv, hd, cap;
  double theta;
  void* q_out;            // [B, nh, S, hd]
  void* k_cache;          // [B, nkv, cap, hd]
  void* v_cache;
  int* err;
};

// Output projection with residual: out[T, N] = x[T, K] . w[N, K]^T (+ residual[T, N]).
struct OprojParams {
  const void* x;          // [T, K]   attention output, heads concatenated (K = nh * hd)
  const void* w;          // [N, K]   W_o, nn.Linear layout
  const void* residual;   // [T, N] or nullptr
  void* out;              // [T, N]   may be the residual itself (in place)
  int T, K, N;
  int* err;
};

// FP8 quantisation of the attention inputs (random-sign Hadamard on q and k).
struct Fp8QuantParams {
  const void* q;          // [B, nh, S, hd] bf16
  const void* k;          // [B, nkv, cap, hd] bf16
  const void* v;
  const int32_t* kv_lens; // [B]
  int B, S, nh, nkv, hd, cap;
  int rotate;             // apply the rotation to q and k
  uint32_t signs[4];      // bit c set: sign of rotation column c is -1
  void* q8;               // [B, nh, S, hd] e4m3
  void* k8;               // [B, nkv, cap, hd] e4m3
  void* v8t;              // [B, nkv, hd, cap] e4m3 (transposed)
  float* amax;            // [3] device: max |value| of rotated q, rotated k, v
  int* err;
};

// FP8 prefill attention over the quantised tensors.
struct Fp8AttnParams {
  const void* q8;         // [B, nh, S, hd] e4m3
  const void* k8;         // [B, nkv, cap, hd] e4m3
  const void* v8t;        // [B, nkv, hd, cap] e4m3
  const float* amax;      // [3] device: the scales are amax / 448
  const int32_t* kv_lens; // [B]
  int B, S, nh, nkv, hd, cap, causal;
  void* out;              // [B, S, nh, hd] bf16
  int* err;
};

struct PrefillParams {
  const void* q;          // [B, nh, S, hd]
  const void* k_cache;    // [B, nkv, cap, hd]
  const void* v_cache;
  const int32_t* q_pos;   // [B, S] or nullptr
  const int32_t* kv_lens; // [B]
  int B, S, nh, nkv, hd, cap, causal;
  void* out;              // [B, S, nh, hd]
  int* err;
  // Packed variable-length mode (cu_q != nullptr): q and out [total_q, nh, hd],
  // k_cache/v_cache [cap, nkv, hd] with cap = total_k; sequence b owns query
  // rows [cu_q[b], cu_q[b+1]) and key rows [cu_k[b], cu_k[b+1]); S is the
  // longest query run (it sizes the grid); q_pos and kv_lens are unused.
  const int32_t* cu_q;
  const int32_t* cu_k;
  int total_q;
  // failure-path testing (gqa_debug_skip_next_kv_tile): K tile + 1 that the
  // first CTA's TMA thread does not load, so that the waits on it run out;
  // 0 = none
  int dbg_skip_tile1;
};

struct DecodeParams {
  const void* q;          // [B, nh, hd]
  const void* k_cache;    // [B, nkv, cap, hd]
  const void* v_cache;
  const int32_t* kv_lens; // [B]
  int B, nh, nkv, hd, cap;
  int split;              // keys per split
  int n_split;            // ceil(cap / split)
  float* ws;              // [B, nh, n_split, hd + 4]: o[hd], m, l, -, -
  void* out;              // [B, nh, hd]
  int* err;
  unsigned* counters;     // [B, nkv, n_hgrp]: finished splits (zero between calls)
  int n_hgrp;             // groups of <= 16 query heads per KV head
  int auto_split;         // the caller left the split to the library
  int cluster;            // set by launch_decode: splits merged inside a thread-block cluster
  // paged cache (block_table != nullptr): k_cache/v_cache are pages
  // [num_pages, nkv, page_size, hd]; key t of sequence b is row t % page_size
  // of page block_table[b * max_pages + t / page_size]; cap = max_pages * page_size
  const int32_t* block_table;
  int page_size, max_pages, num_pages;
};

// Most key splits per sequence: the tensor-core decode's final merge keeps
// (m, l) of every (head row, split) pair in shared memory.
constexpr int kMaxSplits = 512;

constexpr int kWsPad = 4;  // per-partial row: hd floats of o, then m, l and two pad words

// Decode workspace: the counters (rounded up to 256 bytes), then the partials.
inline size_t decode_counter_bytes(int B, int nkv, int n_hgrp) {
  return ((size_t)B * nkv * n_hgrp * sizeof(unsigned) + 255) / 256 * 256;
}
// Tensor-core decode: query heads of a KV head are handled in groups of
// 16 x mtiles.  Measured on B200, two m16 tiles per CTA (233 registers, one
// CTA per SM) made MQA slower than re-reading K/V from L2 for a second group
// of 16 heads, so every group is one tile.
inline int decode_mtiles(int, int) { return 1; }
inline int decode_n_hgrp(int nh, int nkv) {
  const int rows = 16 * decode_mtiles(nh, nkv);
  return (nh / nkv + rows - 1) / rows;
}

// SIMT kernels (any dtype; the fp32 path and shapes the tensor-core kernels skip)
cudaError_t launch_qkv_simt(const QkvParams& p, bool bf16, cudaStream_t st);
cudaError_t launch_prefill_simt(const PrefillParams& p, bool bf16, cudaStream_t st);
cudaError_t launch_decode_simt(const DecodeParams& p, bool bf16, cudaStream_t st);
cudaError_t launch_decode_combine(const DecodeParams& p, bool bf16, cudaStream_t st);

// Tensor-core (tcgen05 + TMA) kernels, bf16 only.
cudaError_t launch_qkv_tc(const QkvParams& p, int num_sms, cudaStream_t st);
cudaError_t launch_qkv_smallm(const QkvParams& p, int num_sms, cudaStream_t st);  // B*S <= 64
// Output projection + residual: tcgen05 GEMM (128-token tiles) and, for at
// most 64 tokens, W-streaming tcgen05 tiles (W rows as M, tokens as N) with
// the reduction dimension split over a thread-block cluster; SIMT for fp32.
cudaError_t launch_oproj_tc(const OprojParams& p, int num_sms, cudaStream_t st);
cudaError_t launch_oproj_smallt(const OprojParams& p, int num_sms, cudaStream_t st);   // T <= 64
// the few-token QKV projection's W-streaming kernel with a residual epilogue
// (T <= 64, K % 64 == 0, N % 16 == 0, tokens' rows fit in shared memory)
bool oproj_stream_fits(const OprojParams& p);
cudaError_t launch_oproj_stream(const OprojParams& p, int num_sms, cudaStream_t st);
cudaError_t launch_oproj_simt(const OprojParams& p, bool bf16, cudaStream_t st);
// FP8 path: amax + quantisation passes, and the tcgen05 kind::f8f6f4 prefill (head_dim 128).
cudaError_t launch_fp8_quantize(const Fp8QuantParams& p, int num_sms, cudaStream_t st);
cudaError_t launch_prefill_fp8(const Fp8AttnParams& p, cudaStream_t st);
// testing aid: tc::exp2_poly2 and exp2f on the same inputs
cudaError_t launch_exp2_check(const float* x, int n, float* poly, float* ref, cudaStream_t st);
cudaError_t launch_prefill_pair(const PrefillParams& p, cudaStream_t st);  // head_dim 64, 2 CTAs/SM
cudaError_t launch_prefill_fa(const PrefillParams& p, cudaStream_t st);    // head_dim 64/128, 2 Q tiles/CTA
cudaError_t launch_decode_mma(const DecodeParams& p, cudaStream_t st);   // head_dim 64 or 128
// tcgen05 decode for large batches with g > 16 (heads as the 128 MMA rows),
// splits merged inside a thread-block cluster (p.n_split <= 8 CTAs);
// decode_tc_splits gives that split count for a problem, or 0 when the
// problem is for the mma.sync kernel.
cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t st);
int decode_tc_splits(const DecodeParams& p);
// tcgen05 decode with the keys as the 128 MMA rows and the heads as N (bf16
// head_dim 128, 16 < g <= 64, the library's split, at least 2^18 cached key
// rows, at most 1024 (sequence, KV head) units): one CTA per SM over equal
// ranges of the units' 128-key tiles.  Its partials take (kHnMaxGrid + units)
// slots of NP x (hd + kWsPad) floats after the counters
// (decode_hn_partial_bytes).
constexpr int kHnMaxGrid = 160;
bool decode_hn_ok(int B, int nh, int nkv, int hd, long long cap, bool auto_split);
size_t decode_hn_partial_bytes(int B, int nh, int nkv);
cudaError_t launch_decode_hn(const DecodeParams& p, cudaStream_t st);

// Decode: for bf16, the tcgen05 cluster decode (contiguous caches it takes,
// g > 16), else the keys-as-rows tcgen05 decode (decode_hn_ok), else the
// mma.sync decode for head_dim 64/128 (the last split of each (sequence, KV
// head, head group) merges the partials itself, using the counters); other
// cases: SIMT partials + the log-sum-exp combine kernel.  Partial m is in log2
// units.  Returns the number of kernels launched; *err the status.
int launch_decode(const DecodeParams& p, bool bf16, cudaStream_t st, cudaError_t* err);

// Raise a kernel's dynamic shared-memory limit on the current device, once per
// device (`done` is the caller's per-kernel flag array), and ask for the
// largest shared-memory carveout: every pipelined kernel of the library then
// runs with the same L1/shared split, so consecutive launches do not make the
// SMs reconfigure it (on B200 a step whose kernels alternated between a small
// and a 215 KB shared-memory configuration lost ~25 us at the switch).  The
// attributes are idempotent, so two threads racing on a first call both set
// them; devices past the array are set on every call.
// Launch with programmatic stream serialization (the kernel calls pdl_wait
// before touching global memory) and, for cluster_x > 1, clusters of
// cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline cudaError_t smem_attr_once(std::atomic<bool> (&done)[64], const void* func, int bytes) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = -1;
  }
  const bool cached = dev >= 0 && dev < 64;
  if (cached && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && cached) done[dev].store(true, std::memory_order_release);
  return e;
}

// 2-D bf16 TMA descriptor with 128-byte swizzle; `map` points at a CUtensorMap.
// Zero fill outside [0, inner) x [0, outer).  False if encoding fails.
bool make_tmap_bf16_2d(void* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                       uint32_t box_inner, uint32_t box_outer);
// 3-D bf16 TMA descriptor with 128-byte swizzle: dims innermost first,
// strides (bytes) of dims 1 and 2, box extents.  Zero fill outside the dims.
bool make_tmap_bf16_3d(void* map, const void* base, const uint64_t dims[3], const uint64_t stride_bytes[2],
                       const uint32_t box[3]);
// Packed token-major rows [tokens, heads, hd] as a 3-D map whose box is one
// head's 64 columns of 128 consecutive tokens: the same swizzled 128 x 64
// tile a 2-D box over head-major rows gives.  tokens == 0 is encoded as 1
// (nothing may then be loaded).
bool make_tmap_packed(void* map, const void* base, uint64_t tokens, int heads, int hd);
// 2-D byte (e4m3) descriptor with 128-byte swizzle, zero fill outside the dims.
bool make_tmap_u8_2d(void* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                     uint32_t box_inner, uint32_t box_outer);

// Shared by the C-ABI translation units (defined in api.cu).
int device_check(int** err);  // GQA_OK, or the status for the current device
void count_launches(int n);
int decode_split_len(int B, int nh, int nkv, int cache_cap, int kv_split);
// Host-side validation shared by the decode entry points (everything but the
// workspace): GQA_OK or the status to return.  B == 0 passes (a no-op).
int decode_check_args(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_lens, int B,
                      int nh, int nkv, int hd, int cap, int kv_split, const void* out, int dtype);
// Decode parameters over a workspace laid out as counters, then partials.
DecodeParams decode_params(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_lens,
                           int B, int nh, int nkv, int hd, int cap, int kv_split, void* out, void* workspace,
                           int* err);

}  // namespace gqa
