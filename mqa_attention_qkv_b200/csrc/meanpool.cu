// MHA -> GQA weight transform ("MHA -> GQA: 提升 LLM 推理效率", section 4.3:
// the new KV projection of each group of heads is initialised by mean pooling
// the group's projections).  An offline step on the fused W_qkv: the query
// rows are copied, each new key (value) row j*hd + d is the mean of rows
// (j*g + i)*hd + d, i < g, of the MHA key (value) block; groups are the
// consecutive heads that attention's head map h -> h / g gives one KV head.
//
// Memory-bound: each input row is read once and each output row written once
// (algorithmic bytes = (3 nh + nh + 2 nkv) hd D x element size).  A thread
// takes one 16-byte vector of an output row; the g source vectors of a KV row
// are independent loads, summed in fp32 and rounded once.  Grid-stride over
// all output vectors, sized to a few CTAs per SM.
#include "common.cuh"
#include "kernels.h"

namespace gqa {
namespace {

template <bool BF16>
struct Vec;
template <>
struct Vec<true> {  // 8 bf16
  static constexpr int N = 8;
  using T = __nv_bfloat16;
};
template <>
struct Vec<false> {  // 4 float
  static constexpr int N = 4;
  using T = float;
};

template <bool BF16>
__device__ __forceinline__ void load_vec(const void* p, float (&v)[Vec<BF16>::N]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  if (BF16) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
  }
}

template <bool BF16>
__device__ __forceinline__ void store_vec(void* p, const float (&v)[Vec<BF16>::N]) {
  uint4 u;
  if (BF16) {
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    u.z = pack_bf16x2(v[4], v[5]);
    u.w = pack_bf16x2(v[6], v[7]);
  } else {
    u = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
  }
  *reinterpret_cast<uint4*>(p) = u;
}

template <bool BF16>
__global__ void __launch_bounds__(256) meanpool_kernel(const void* __restrict__ w_in, void* __restrict__ w_out, int nh,
                                                       int nkv, int hd, int D, long long n_vec) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  using V = Vec<BF16>;
  using T = typename V::T;
  const T* in = static_cast<const T*>(w_in);
  T* out = static_cast<T*>(w_out);
  const int vpr = D / V::N;  // vectors per row
  const int g = nh / nkv;
  const float inv_g = 1.f / (float)g;
  const long long q_rows = (long long)nh * hd, kv_rows = (long long)nkv * hd;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n_vec;
       e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / vpr;
    const int c = (int)(e - r * vpr) * V::N;
    float acc[V::N];
    if (r < q_rows) {  // query projection: kept
      load_vec<BF16>(in + r * D + c, acc);
    } else {
      const long long rr = r - q_rows;
      const int block = (int)(rr / kv_rows);  // 0: key, 1: value
      const int jd = (int)(rr - block * kv_rows), j = jd / hd, d = jd - j * hd;
      const T* src = in + ((1 + block) * q_rows + (long long)j * g * hd + d) * D + c;
#pragma unroll
      for (int i = 0; i < V::N; ++i) acc[i] = 0.f;
      for (int k = 0; k < g; ++k) {
        float v[V::N];
        load_vec<BF16>(src + (long long)k * hd * D, v);
#pragma unroll
        for (int i = 0; i < V::N; ++i) acc[i] += v[i];
      }
#pragma unroll
      for (int i = 0; i < V::N; ++i) acc[i] *= inv_g;
    }
    store_vec<BF16>(out + r * D + c, acc);
  }
}

}  // namespace
}  // namespace gqa

extern "C" int gqa_meanpool_kv_heads(const void* w_qkv_mha, int hidden, int n_heads, int n_kv_heads,
                                     int head_dim, void* w_qkv_gqa, int dtype, void* stream) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED_DTYPE;
  if (hidden <= 0 || n_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0) return GQA_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads != 0) return GQA_ERR_INVALID_ARG;
  if (!w_qkv_mha || !w_qkv_gqa) return GQA_ERR_INVALID_ARG;
  const int vec = dtype == GQA_BF16 ? 8 : 4;  // elements per 16-byte vector
  if (hidden % vec) return GQA_ERR_UNSUPPORTED_SHAPE;
  if ((long long)3 * n_heads * head_dim * hidden > (1ll << 40)) return GQA_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(w_qkv_mha) & 15u) || (reinterpret_cast<uintptr_t>(w_qkv_gqa) & 15u))
    return GQA_ERR_MISALIGNED;
  const size_t esz = dtype == GQA_BF16 ? 2 : 4;
  const char* ib = static_cast<const char*>(w_qkv_mha);
  const char* ob = static_cast<const char*>(w_qkv_gqa);
  const size_t in_bytes = (size_t)3 * n_heads * head_dim * hidden * esz;
  const size_t out_bytes = (size_t)(n_heads + 2 * n_kv_heads) * head_dim * hidden * esz;
  if (ib < ob + out_bytes && ob < ib + in_bytes) return GQA_ERR_INVALID_ARG;  // the buffers overlap
  int* err = nullptr;
  const int st = gqa::device_check(&err);
  if (st != GQA_OK) return st;
  const long long n_vec = (long long)(n_heads + 2 * n_kv_heads) * head_dim * (hidden / vec);
  long long grid = (n_vec + 255) / 256;
  if (grid > 148 * 8) grid = 148 * 8;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e =
      dtype == GQA_BF16
          ? gqa::launch_ex(gqa::meanpool_kernel<true>, dim3((unsigned)grid), dim3(256), 0, s, 1u, w_qkv_mha, w_qkv_gqa,
                           n_heads, n_kv_heads, head_dim, hidden, n_vec)
          : gqa::launch_ex(gqa::meanpool_kernel<false>, dim3((unsigned)grid), dim3(256), 0, s, 1u, w_qkv_mha, w_qkv_gqa,
                           n_heads, n_kv_heads, head_dim, hidden, n_vec);
  gqa::count_launches(1);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_LAUNCH_FAILED;
  }
  return GQA_OK;
}
