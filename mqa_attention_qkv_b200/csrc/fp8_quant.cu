// FP8 (e4m3) quantisation of the attention inputs with incoherent processing
// (FlashAttention-3 summary, section "FP8低精度とincoherent processing"):
// query and key rows are multiplied by one random-sign Hadamard rotation
// M = H diag(s) / sqrt(hd) (H the Sylvester Hadamard matrix), which spreads
// outlier features over the whole row and leaves every score q.k unchanged,
// then q, k and v are each scaled by 448 / amax of the tensor and rounded to
// e4m3 (nearest, ties to even, saturating).  V is not rotated.
//
// Two passes over the bf16 inputs, both memory-bound:
//   amax      warp = one row of hd elements; the rotation is a fast
//             Walsh-Hadamard transform in registers and warp shuffles (the
//             lane holds hd/32 consecutive elements: in-lane butterflies for
//             the small strides, __shfl_xor for the others); per-warp maxima
//             go to the three scale slots with an integer atomicMax on the
//             (non-negative) float bits
//   quantise  the same rows again: rotate, scale, round.  q and k keep their
//             row layout; v is written transposed per (sequence, KV head),
//             [hd, cap], so that the FP8 attention can read it K-major for
//             P.V: a CTA takes 64 cache slots of one (b, j), quantises them
//             into shared memory and stores 64-byte runs of each hd row.
// Cache rows at or beyond a sequence's kv_len are never read (they may hold
// NaN) and are written as zeros.
#include "kernels.h"
#include "common.cuh"

namespace gqa {
namespace {

constexpr float kE4m3Max = 448.0f;

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// The lane's hd/32 consecutive elements of row `src` (bf16), rotated when
// `rotate`: y = FWHT(x) * s / sqrt(hd).
template <int HD>
__device__ __forceinline__ void load_row(const __nv_bfloat16* src, bool valid, bool rotate, const uint32_t (&signs)[4],
                                         float (&y)[HD / 32]) {
  constexpr int E = HD / 32;
  const int lane = threadIdx.x & 31;
  if (valid) {
    if (E == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(src + 4 * lane);
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
      y[0] = __low2float(a);
      y[1] = __high2float(a);
      y[2 % E] = __low2float(b);
      y[3 % E] = __high2float(b);
    } else {
      const uint32_t u = *reinterpret_cast<const uint32_t*>(src + 2 * lane);
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u);
      y[0] = __low2float(a);
      y[1 % E] = __high2float(a);
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) y[e] = 0.f;
  }
  if (!rotate) return;
  // in-lane strides 1 .. E/2
#pragma unroll
  for (int h = 1; h < E; h *= 2)
#pragma unroll
    for (int i = 0; i < E; ++i)
      if (!(i & h)) {
        const float a = y[i], b = y[i + h];
        y[i] = a + b;
        y[i + h] = a - b;
      }
  // cross-lane strides E .. HD/2: partner lane = lane ^ (h / E)
#pragma unroll
  for (int h = E; h < HD; h *= 2) {
    const bool upper = (lane * E) & h;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, y[i], h / E);
      y[i] = upper ? o - y[i] : y[i] + o;
    }
  }
  const float inv_sqrt = rsqrtf((float)HD);
  // the lane's E sign bits sit in one 32-bit word (E divides 32)
  const int wi = (lane * E) >> 5;
  const uint32_t word = wi == 0 ? signs[0] : wi == 1 ? signs[1] : wi == 2 ? signs[2] : signs[3];
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const bool neg = (word >> ((lane * E + i) & 31)) & 1u;
    y[i] = (neg ? -y[i] : y[i]) * inv_sqrt;
  }
}

// Row r of the three tensors: q rows first, then k rows, then v rows.
struct RowRef {
  const __nv_bfloat16* src;
  int tensor;      // 0 q, 1 k, 2 v
  bool valid;
  long long row;   // row index inside its tensor
};

__device__ __forceinline__ RowRef row_ref(const Fp8QuantParams& p, long long r) {
  RowRef rr;
  const long long nq = (long long)p.B * p.nh * p.S, nc = (long long)p.B * p.nkv * p.cap;
  if (r < nq) {
    rr.tensor = 0;
    rr.row = r;
    rr.valid = true;
    rr.src = static_cast<const __nv_bfloat16*>(p.q) + r * p.hd;
    return rr;
  }
  r -= nq;
  rr.tensor = r < nc ? 1 : 2;
  if (r >= nc) r -= nc;
  rr.row = r;
  const int b = (int)(r / ((long long)p.nkv * p.cap));
  const int slot = (int)(r % p.cap);
  int len = p.kv_lens[b];
  len = len < 0 ? 0 : (len > p.cap ? p.cap : len);
  rr.valid = slot < len;
  rr.src = static_cast<const __nv_bfloat16*>(rr.tensor == 1 ? p.k : p.v) + r * p.hd;
  return rr;
}

template <int HD>
__global__ void __launch_bounds__(256) fp8_amax_kernel(Fp8QuantParams p, long long n_rows) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  constexpr int E = HD / 32;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const long long nwarps = (long long)gridDim.x * blockDim.x / 32;
  float m0 = 0.f, m1 = 0.f, m2 = 0.f;
  for (long long r = warp0; r < n_rows; r += nwarps) {
    const RowRef rr = row_ref(p, r);
    float y[E];
    load_row<HD>(rr.src, rr.valid, rr.tensor < 2 && p.rotate, p.signs, y);
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < E; ++i) a = fmaxf(a, fabsf(y[i]));
    if (rr.tensor == 0) m0 = fmaxf(m0, a);
    else if (rr.tensor == 1) m1 = fmaxf(m1, a);
    else m2 = fmaxf(m2, a);
  }
#pragma unroll
  for (int t = 0; t < 3; ++t) {
    float a = t == 0 ? m0 : t == 1 ? m1 : m2;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0 && a > 0.f) atomicMax(reinterpret_cast<unsigned*>(p.amax) + t, __float_as_uint(a));
  }
}

__device__ __forceinline__ float inv_scale(const float* amax, int t) {
  const float a = amax[t];
  return a > 0.f ? kE4m3Max / a : 1.f;
}

// q and k rows -> e4m3 rows (rotated)
template <int HD>
__global__ void __launch_bounds__(256) fp8_quant_qk_kernel(Fp8QuantParams p, long long n_rows) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  constexpr int E = HD / 32;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const long long nwarps = (long long)gridDim.x * blockDim.x / 32;
  const int lane = threadIdx.x & 31;
  const float inv_q = inv_scale(p.amax, 0), inv_k = inv_scale(p.amax, 1);
  for (long long r = warp0; r < n_rows; r += nwarps) {
    const RowRef rr = row_ref(p, r);
    float y[E];
    load_row<HD>(rr.src, rr.valid, p.rotate, p.signs, y);
    uint8_t* dst = static_cast<uint8_t*>(rr.tensor == 0 ? p.q8 : p.k8) + rr.row * HD + lane * E;
    const float s = rr.tensor == 0 ? inv_q : inv_k;
    if (E == 4) {
      const uint32_t w = (uint32_t)e4m3x2(y[0] * s, y[1 % E] * s) | ((uint32_t)e4m3x2(y[2 % E] * s, y[3 % E] * s) << 16);
      *reinterpret_cast<uint32_t*>(dst) = rr.valid ? w : 0u;
    } else {
      const uint16_t w = e4m3x2(y[0] * s, y[1 % E] * s);
      *reinterpret_cast<uint16_t*>(dst) = rr.valid ? w : (uint16_t)0;
    }
  }
}

// v rows -> e4m3, transposed per (b, j) to [hd, cap]; CTA = 64 slots of one (b, j)
template <int HD>
__global__ void __launch_bounds__(256) fp8_quant_v_kernel(Fp8QuantParams p, int slot_tiles) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  constexpr int E = HD / 32, SLOTS = 64;
  __shared__ uint8_t tile[HD][SLOTS + 4];
  const int bj = blockIdx.x / slot_tiles, s0 = (blockIdx.x % slot_tiles) * SLOTS;
  const int b = bj / p.nkv;
  int len = p.kv_lens[b];
  len = len < 0 ? 0 : (len > p.cap ? p.cap : len);
  const float s = inv_scale(p.amax, 2);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const uint32_t none[4] = {0u, 0u, 0u, 0u};
  for (int i = warp; i < SLOTS; i += 8) {
    const int slot = s0 + i;
    const bool valid = slot < len;
    float y[E];
    load_row<HD>(static_cast<const __nv_bfloat16*>(p.v) + ((long long)bj * p.cap + (slot < p.cap ? slot : 0)) * HD,
                 valid, false, none, y);
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const uint16_t w = valid ? e4m3x2(y[e] * s, y[(e + 1) % E] * s) : (uint16_t)0;
      tile[lane * E + e][i] = (uint8_t)(w & 0xFF);
      tile[lane * E + e + 1][i] = (uint8_t)(w >> 8);
    }
  }
  __syncthreads();
  // each hd row: 64 bytes at [bj, c, s0 .. s0 + 63] (cap % 16 == 0 keeps them aligned)
  uint8_t* dst = static_cast<uint8_t*>(p.v8t) + (long long)bj * HD * p.cap + s0;
  const int n = min(SLOTS, p.cap - s0);
  for (int e = threadIdx.x; e < HD * (SLOTS / 16); e += 256) {
    const int c = e / (SLOTS / 16), ch = e % (SLOTS / 16);
    if (ch * 16 >= n) continue;
    uint4 v;
    uint8_t* vb = reinterpret_cast<uint8_t*>(&v);
#pragma unroll
    for (int k = 0; k < 16; ++k) vb[k] = tile[c][ch * 16 + k];
    *reinterpret_cast<uint4*>(dst + (long long)c * p.cap + ch * 16) = v;
  }
}

template <int HD>
cudaError_t launch_hd(const Fp8QuantParams& p, int num_sms, cudaStream_t st) {
  if (cudaError_t e = cudaMemsetAsync(p.amax, 0, 3 * sizeof(float), st); e != cudaSuccess) return e;
  const long long nq = (long long)p.B * p.nh * p.S, nc = (long long)p.B * p.nkv * p.cap;
  const long long rows = nq + 2 * nc;
  long long blocks = (rows + 7) / 8;
  if (blocks > (long long)num_sms * 16) blocks = (long long)num_sms * 16;
  if (cudaError_t e = launch_ex(fp8_amax_kernel<HD>, dim3((unsigned)blocks), dim3(256), 0, st, 1u, p, rows);
      e != cudaSuccess)
    return e;
  long long qk_blocks = (nq + nc + 7) / 8;
  if (qk_blocks > (long long)num_sms * 16) qk_blocks = (long long)num_sms * 16;
  if (cudaError_t e = launch_ex(fp8_quant_qk_kernel<HD>, dim3((unsigned)qk_blocks), dim3(256), 0, st, 1u, p, nq + nc);
      e != cudaSuccess)
    return e;
  const int slot_tiles = (p.cap + 63) / 64;
  return launch_ex(fp8_quant_v_kernel<HD>, dim3((unsigned)((long long)p.B * p.nkv * slot_tiles)), dim3(256), 0, st, 1u,
                   p, slot_tiles);
}

}  // namespace

cudaError_t launch_fp8_quantize(const Fp8QuantParams& p, int num_sms, cudaStream_t st) {
  switch (p.hd) {
    case 64: return launch_hd<64>(p, num_sms, st);
    case 128: return launch_hd<128>(p, num_sms, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gqa
