// SIMT (FFMA) kernels: the float32 path of all three calls, and the general
// shapes the tensor-core kernels do not take.
//
//  qkv_simt        fused projection tile [32 tokens x one head] with the RoPE
//                  rotation and the head-major scatter in its epilogue
//  attn_simt       online-softmax attention over key tiles of 32 for up to 16
//                  query rows that share one KV head (prefill: 16 query
//                  positions of one head; decode: 16 of the g heads of one KV
//                  head over one key split, writing an unnormalised partial)
//  decode_combine  log-sum-exp merge of the decode partials
//  oproj_simt      output projection + residual, one output element per
//                  thread (float32, and bf16 widths the tensor path skips)
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace gqa {
namespace {

// ---------------------------------------------------------------------------
// qkv_simt: Y = X W^T for a 32-token x HD-feature tile (one head of the fused
// width), then RoPE on q/k heads and the scatter.
// Thread (i, rg) owns feature pair (i, i + HD/2) for rows rg, rg + NRG, ...
// so the rotation needs no data exchange.
// ---------------------------------------------------------------------------
template <typename T, int HD>
__global__ void __launch_bounds__(256) qkv_simt_kernel(QkvParams p) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  constexpr int BM = 32, BK = 32, HALF = HD / 2, NRG = 256 / HALF, RPT = BM / NRG;
  __shared__ float xs[BM][BK + 1];
  __shared__ float ws[HD][BK + 1];

  const int tid = threadIdx.x;
  const int i = tid % HALF, rg = tid / HALF;
  const int T_tot = p.B * p.S;
  const int t0 = blockIdx.x * BM;
  const int hb = blockIdx.y;  // head block of the fused output
  const T* x = static_cast<const T*>(p.x);
  const T* w = static_cast<const T*>(p.w);
  const size_t wrow0 = (size_t)hb * HD;

  float acc_lo[RPT], acc_hi[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) acc_lo[r] = acc_hi[r] = 0.f;

  for (int k0 = 0; k0 < p.hidden; k0 += BK) {
    for (int e = tid; e < BM * BK; e += 256) {
      int r = e / BK, k = e % BK;
      int t = t0 + r, kk = k0 + k;
      xs[r][k] = (t < T_tot && kk < p.hidden) ? to_f32(x[(size_t)t * p.hidden + kk]) : 0.f;
    }
    for (int e = tid; e < HD * BK; e += 256) {
      int n = e / BK, k = e % BK;
      int kk = k0 + k;
      ws[n][k] = (kk < p.hidden) ? to_f32(w[(wrow0 + n) * p.hidden + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < BK; ++k) {
      const float wl = ws[i][k], wh = ws[i + HALF][k];
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const float xv = xs[rg + r * NRG][k];
        acc_lo[r] = fmaf(xv, wl, acc_lo[r]);
        acc_hi[r] = fmaf(xv, wh, acc_hi[r]);
      }
    }
    __syncthreads();
  }

  const bool is_q = hb < p.nh, is_k = !is_q && hb < p.nh + p.nkv;
  const double inv_freq = rope_inv_freq(i, HD, p.theta);
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int t = t0 + rg + r * NRG;
    if (t >= T_tot) continue;
    const int b = t / p.S, s = t % p.S;
    const int pos = p.pos[t];
    float lo = acc_lo[r], hi = acc_hi[r];
    if (is_q || is_k) {
      float c, sn;
      rope_cos_sin(pos, inv_freq, &c, &sn);
      const float nlo = lo * c - hi * sn;
      const float nhi = hi * c + lo * sn;
      lo = nlo;
      hi = nhi;
    }
    T* dst;
    if (is_q) {
      dst = static_cast<T*>(p.q_out) + (((size_t)b * p.nh + hb) * p.S + s) * HD;
    } else {
      if (pos < 0 || pos >= p.cap) {
        if (i == 0) raise_error(p.err, GQA_DEVERR_POSITION_RANGE);
        continue;
      }
      const int j = is_k ? hb - p.nh : hb - p.nh - p.nkv;
      T* base = static_cast<T*>(is_k ? p.k_cache : p.v_cache);
      dst = base + (((size_t)b * p.nkv + j) * p.cap + pos) * HD;
    }
    dst[i] = from_f32<T>(lo);
    dst[i + HALF] = from_f32<T>(hi);
  }
}

// ---------------------------------------------------------------------------
// attn_simt: 4 warps x 4 rows.  Per key tile of 32: lane t scores key t for a
// row, the warp takes the max/sum, and each lane accumulates HD/32 output
// features over the tile's keys (p_t broadcast by shuffle).
// ---------------------------------------------------------------------------
constexpr int kRows = 16, kKT = 32;

template <typename T>
__device__ __forceinline__ float round_p(float v) { return v; }
template <>
__device__ __forceinline__ float round_p<__nv_bfloat16>(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

template <typename T, int HD, bool DECODE>
__global__ void __launch_bounds__(128) attn_simt_kernel(PrefillParams pp, DecodeParams dp) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  constexpr int PER = HD / 32;
  __shared__ float qs[kRows][HD];
  __shared__ float ks[kKT][HD + 1];
  __shared__ float vs[kKT][HD];
  __shared__ int row_hi[kRows];
  __shared__ int tile_hi;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = blockIdx.z, j = blockIdx.y;
  const int nh = DECODE ? dp.nh : pp.nh, nkv = DECODE ? dp.nkv : pp.nkv;
  const int cap = DECODE ? dp.cap : pp.cap;
  const int g = nh / nkv;
  int* err = DECODE ? dp.err : pp.err;

  int kv_len = DECODE ? dp.kv_lens[b] : pp.kv_lens[b];
  if (kv_len > cap || kv_len < 0) {
    if (threadIdx.x == 0) raise_error(err, GQA_DEVERR_KVLEN_RANGE);
    kv_len = kv_len > cap ? cap : 0;
  }

  // Rows of this block and the key range they share.
  int k_lo = 0, k_hi;
  int split = 0, hgrp = 0, h_fixed = 0, s0 = 0;
  if (DECODE) {
    const int n_hgrp = (g + kRows - 1) / kRows;
    split = blockIdx.x / n_hgrp;
    hgrp = blockIdx.x % n_hgrp;
    k_lo = split * dp.split;
    k_hi = min(kv_len, k_lo + dp.split);
    if (k_lo >= kv_len) return;  // this split holds no key of the sequence
  } else {
    h_fixed = j;  // prefill grid.y is the query head
    s0 = blockIdx.x * kRows;
    k_hi = 0;
  }

  // Load q rows and per-row visible limits.
  for (int e = threadIdx.x; e < kRows * HD; e += 128) {
    const int r = e / HD, d = e % HD;
    float v = 0.f;
    if (DECODE) {
      const int hl = hgrp * kRows + r;
      if (hl < g) {
        const int h = (blockIdx.y) * g + hl;
        v = to_f32(static_cast<const T*>(dp.q)[((size_t)b * nh + h) * HD + d]);
      }
    } else {
      const int s = s0 + r;
      if (s < pp.S) v = to_f32(static_cast<const T*>(pp.q)[(((size_t)b * nh + h_fixed) * pp.S + s) * HD + d]);
    }
    qs[r][d] = v;
  }
  if (threadIdx.x < kRows) {
    const int r = threadIdx.x;
    int hi = 0;
    if (DECODE) {
      hi = (hgrp * kRows + r < g) ? k_hi : 0;
    } else {
      const int s = s0 + r;
      if (s < pp.S) {
        const int pos = pp.q_pos ? pp.q_pos[(size_t)b * pp.S + s] : kv_len - pp.S + s;
        hi = pp.causal ? max(0, min(kv_len, pos + 1)) : kv_len;
      }
    }
    row_hi[r] = hi;
  }
  __syncthreads();
  if (!DECODE) {
    if (threadIdx.x == 0) {
      int m = 0;
      for (int r = 0; r < kRows; ++r) m = max(m, row_hi[r]);
      tile_hi = m;
    }
    __syncthreads();
    k_hi = tile_hi;
  }

  const int kvh = DECODE ? j : h_fixed / g;
  const T* kc = static_cast<const T*>(DECODE ? dp.k_cache : pp.k_cache) + ((size_t)b * nkv + kvh) * cap * HD;
  const T* vc = static_cast<const T*>(DECODE ? dp.v_cache : pp.v_cache) + ((size_t)b * nkv + kvh) * cap * HD;
  const float scale = rsqrtf((float)HD);

  float m_r[4], l_r[4], acc[4][PER];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    m_r[r] = -INFINITY;
    l_r[r] = 0.f;
#pragma unroll
    for (int d = 0; d < PER; ++d) acc[r][d] = 0.f;
  }

  for (int t0 = k_lo; t0 < k_hi; t0 += kKT) {
    for (int e = threadIdx.x; e < kKT * HD; e += 128) {
      const int t = e / HD, d = e % HD;
      const bool ok = t0 + t < k_hi;
      ks[t][d] = ok ? to_f32(kc[(size_t)(t0 + t) * HD + d]) : 0.f;
      vs[t][d] = ok ? to_f32(vc[(size_t)(t0 + t) * HD + d]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = warp * 4 + rr;
      const int hi = row_hi[r];
      if (t0 >= hi) continue;  // warp-uniform
      const int t = t0 + lane;
      float sc = 0.f;
#pragma unroll 8
      for (int d = 0; d < HD; ++d) sc = fmaf(qs[r][d], ks[lane][d], sc);
      sc = (t < hi) ? sc * scale : -INFINITY;
      float mx = sc;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m_r[rr], mx);
      const float alpha = expf(m_r[rr] - m_new);  // m_r = -inf on the first tile -> 0
      const float pr = (t < hi) ? expf(sc - m_new) : 0.f;
      float sum = pr;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      l_r[rr] = l_r[rr] * alpha + sum;
      m_r[rr] = m_new;
      const float pv_w = round_p<T>(pr);
#pragma unroll
      for (int d = 0; d < PER; ++d) acc[rr][d] *= alpha;
      for (int tt = 0; tt < kKT; ++tt) {
        const float pt = __shfl_sync(0xffffffffu, pv_w, tt);
#pragma unroll
        for (int d = 0; d < PER; ++d) acc[rr][d] = fmaf(pt, vs[tt][lane + 32 * d], acc[rr][d]);
      }
    }
    __syncthreads();
  }

  // Write results.
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = warp * 4 + rr;
    if (DECODE) {
      const int hl = hgrp * kRows + r;
      if (hl >= g) continue;
      const int h = j * g + hl;
      float* row = dp.ws + (((size_t)b * nh + h) * dp.n_split + split) * (HD + kWsPad);
#pragma unroll
      for (int d = 0; d < PER; ++d) row[lane + 32 * d] = acc[rr][d];
      if (lane == 0) {
        row[HD] = m_r[rr] * 1.4426950408889634f;  // partial max in log2 units
        row[HD + 1] = l_r[rr];
      }
    } else {
      const int s = s0 + r;
      if (s >= pp.S) continue;
      const float inv = l_r[rr] > 0.f ? 1.f / l_r[rr] : 0.f;
      T* o = static_cast<T*>(pp.out) + (((size_t)b * pp.S + s) * nh + h_fixed) * HD;
#pragma unroll
      for (int d = 0; d < PER; ++d) o[lane + 32 * d] = from_f32<T>(acc[rr][d] * inv);
    }
  }
}

// ---------------------------------------------------------------------------
// decode_combine: one warp per (b, h).  Partials c = 0..n-1 with n =
// ceil(kv_len / split), their maxima m_c in log2 units of the scaled score;
// M = max m_c, L = sum l_c 2^(m_c - M), O = sum o_c 2^(m_c - M) / L.
// ---------------------------------------------------------------------------
template <typename T, int HD>
__global__ void __launch_bounds__(128) decode_combine_kernel(DecodeParams p) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  constexpr int PER = HD / 32;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const size_t row = (size_t)blockIdx.x * 4 + warp;
  if (row >= (size_t)p.B * p.nh) return;
  const int b = (int)(row / p.nh);
  int kv_len = p.kv_lens[b];
  kv_len = kv_len > p.cap ? p.cap : (kv_len < 0 ? 0 : kv_len);
  const int n = (kv_len + p.split - 1) / p.split;
  const float* ws = p.ws + row * p.n_split * (HD + kWsPad);

  float M = -INFINITY;
  for (int c = 0; c < n; ++c) M = fmaxf(M, ws[(size_t)c * (HD + kWsPad) + HD]);
  float L = 0.f, o[PER];
#pragma unroll
  for (int d = 0; d < PER; ++d) o[d] = 0.f;
  if (M != -INFINITY) {
    for (int c = 0; c < n; ++c) {
      const float* part = ws + (size_t)c * (HD + kWsPad);
      const float e = exp2f(part[HD] - M);
      L += part[HD + 1] * e;
#pragma unroll
      for (int d = 0; d < PER; ++d) o[d] = fmaf(part[lane + 32 * d], e, o[d]);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  T* out = static_cast<T*>(p.out) + row * HD;
#pragma unroll
  for (int d = 0; d < PER; ++d) out[lane + 32 * d] = from_f32<T>(o[d] * inv);
}

// ---------------------------------------------------------------------------
// oproj_simt: out[t, n] = sum_k x[t, k] w[n, k] (+ residual[t, n]); a block of
// 128 threads takes 128 consecutive outputs n of one token t and stages the
// token's row of x through shared memory in chunks.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) oproj_simt_kernel(OprojParams p) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  constexpr int CH = 256;
  __shared__ float xs[CH];
  const int n = blockIdx.x * 128 + threadIdx.x;
  const T* w = static_cast<const T*>(p.w) + (size_t)(n < p.N ? n : 0) * p.K;
  for (int t = blockIdx.y; t < p.T; t += gridDim.y) {
    const T* x = static_cast<const T*>(p.x) + (size_t)t * p.K;
    float acc = 0.f;
    for (int k0 = 0; k0 < p.K; k0 += CH) {
      const int kn = min(CH, p.K - k0);
      __syncthreads();
      for (int k = threadIdx.x; k < kn; k += 128) xs[k] = to_f32(x[k0 + k]);
      __syncthreads();
      if (n < p.N)
        for (int k = 0; k < kn; ++k) acc = fmaf(xs[k], to_f32(w[k0 + k]), acc);
    }
    if (n < p.N) {
      const size_t o = (size_t)t * p.N + n;
      if (p.residual) acc += to_f32(static_cast<const T*>(p.residual)[o]);
      static_cast<T*>(p.out)[o] = from_f32<T>(acc);
    }
  }
}

template <typename T>
cudaError_t qkv_dispatch(const QkvParams& p, cudaStream_t st) {
  const int T_tot = p.B * p.S;
  dim3 grid((T_tot + 31) / 32, p.nh + 2 * p.nkv);
  switch (p.hd) {
    case 32: return launch_ex(qkv_simt_kernel<T, 32>, dim3(grid), dim3(256), 0, st, 1u, p);
    case 64: return launch_ex(qkv_simt_kernel<T, 64>, dim3(grid), dim3(256), 0, st, 1u, p);
    case 128: return launch_ex(qkv_simt_kernel<T, 128>, dim3(grid), dim3(256), 0, st, 1u, p);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, bool DECODE>
cudaError_t attn_dispatch(const PrefillParams& pp, const DecodeParams& dp, dim3 grid, int hd,
                          cudaStream_t st) {
  switch (hd) {
    case 32: return launch_ex(attn_simt_kernel<T, 32, DECODE>, dim3(grid), dim3(128), 0, st, 1u, pp, dp);
    case 64: return launch_ex(attn_simt_kernel<T, 64, DECODE>, dim3(grid), dim3(128), 0, st, 1u, pp, dp);
    case 128: return launch_ex(attn_simt_kernel<T, 128, DECODE>, dim3(grid), dim3(128), 0, st, 1u, pp, dp);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t combine_dispatch(const DecodeParams& p, cudaStream_t st) {
  dim3 grid((unsigned)(((size_t)p.B * p.nh + 3) / 4));
  switch (p.hd) {
    case 32: return launch_ex(decode_combine_kernel<T, 32>, dim3(grid), dim3(128), 0, st, 1u, p);
    case 64: return launch_ex(decode_combine_kernel<T, 64>, dim3(grid), dim3(128), 0, st, 1u, p);
    case 128: return launch_ex(decode_combine_kernel<T, 128>, dim3(grid), dim3(128), 0, st, 1u, p);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_qkv_simt(const QkvParams& p, bool bf16, cudaStream_t st) {
  return bf16 ? qkv_dispatch<__nv_bfloat16>(p, st) : qkv_dispatch<float>(p, st);
}

cudaError_t launch_prefill_simt(const PrefillParams& p, bool bf16, cudaStream_t st) {
  dim3 grid((p.S + kRows - 1) / kRows, p.nh, p.B);
  DecodeParams none{};
  return bf16 ? attn_dispatch<__nv_bfloat16, false>(p, none, grid, p.hd, st)
              : attn_dispatch<float, false>(p, none, grid, p.hd, st);
}

cudaError_t launch_decode_simt(const DecodeParams& p, bool bf16, cudaStream_t st) {
  const int g = p.nh / p.nkv;
  const int n_hgrp = (g + kRows - 1) / kRows;
  dim3 grid(p.n_split * n_hgrp, p.nkv, p.B);
  PrefillParams none{};
  return bf16 ? attn_dispatch<__nv_bfloat16, true>(none, p, grid, p.hd, st)
              : attn_dispatch<float, true>(none, p, grid, p.hd, st);
}

cudaError_t launch_oproj_simt(const OprojParams& p, bool bf16, cudaStream_t st) {
  dim3 grid((unsigned)((p.N + 127) / 128), (unsigned)(p.T < 65535 ? p.T : 65535));
  if (bf16) return launch_ex(oproj_simt_kernel<__nv_bfloat16>, dim3(grid), dim3(128), 0, st, 1u, p);
  return launch_ex(oproj_simt_kernel<float>, dim3(grid), dim3(128), 0, st, 1u, p);
}

namespace {
// testing aid: the prefill softmax's polynomial 2^x next to CUDA's exp2f
__global__ void exp2_check_kernel(const float* x, int n, float* poly, float* ref) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
  const float ra = exp2f(a), rb = exp2f(b);
  tc::exp2_poly2(a, b);
  poly[i] = a;
  ref[i] = ra;
  if (i + 1 < n) {
    poly[i + 1] = b;
    ref[i + 1] = rb;
  }
}
}  // namespace

cudaError_t launch_exp2_check(const float* x, int n, float* poly, float* ref, cudaStream_t st) {
  exp2_check_kernel<<<(unsigned)((n + 511) / 512), 256, 0, st>>>(x, n, poly, ref);
  return cudaGetLastError();
}

cudaError_t launch_decode_combine(const DecodeParams& p, bool bf16, cudaStream_t st) {
  return bf16 ? combine_dispatch<__nv_bfloat16>(p, st) : combine_dispatch<float>(p, st);
}

}  // namespace gqa
