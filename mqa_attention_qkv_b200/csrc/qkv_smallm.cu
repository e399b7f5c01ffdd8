// Fused QKV projection for a handful of tokens (T <= 64: the one-token decode
// steps of a generation loop), with the same RoPE + head-major scatter
// epilogue as the big tensor-core GEMM (steps a1-a3, bf16).
//
// With T tokens of hidden size D the projection reads the whole W_qkv
// (N x D) to do 2*T*N*D flops: it is bound by the W stream (the "batch-1 is
// matrix-vector, memory-bound" case of the MHA -> GQA blog, section 3.1), so
// the design goal is to spread W over every SM with many bytes in flight.
//
// CTA = 16 rows of W: 8 consecutive features at offset i0 of the first half
// of one head and the 8 features i0 + hd/2 of its second half, i.e. 8 RoPE
// pairs, so the rotation happens inside the CTA.  8 warps split D; each
// thread streams 16-byte vectors of its W rows (no L1 allocation) and of the
// tokens' hidden states straight into mma.sync m16n8k16 fragments (W rows as
// M, tokens as N).  Inside every 32-element K block the 16-byte chunk of
// thread tq holds elements 8tq..8tq+7; those are assigned to the fragment
// k-slots 2tq, 2tq+1, 2tq+8, 2tq+9 of two consecutive k16 steps for both
// operands, so W and X agree on which K element each slot holds.  The 8
// warps' accumulators are summed through shared memory, then 64 threads
// rotate and store the 8 pairs for every token.
#include "kernels.h"
#include "tc.cuh"

namespace gqa {
namespace {

constexpr int WARPS = 8;

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ldg_keep(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int NT, int HD>
__global__ void __launch_bounds__(WARPS * 32, 2) qkv_smallm_kernel(QkvParams p) {
  constexpr int U = NT == 1 ? 8 : (NT == 2 ? 4 : 2);   // K blocks in flight per thread
  constexpr int TP = NT * 8;                            // padded token count
  __shared__ float red[WARPS][16][TP + 1];
  __shared__ double inv_freq[8];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane >> 2, tq = lane & 3;
  constexpr int GROUPS = HD / 16;
  const int hb = blockIdx.x / GROUPS, i0 = (blockIdx.x % GROUPS) * 8;
  const int T = p.B * p.S, D = p.hidden;
  const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(p.w);
  const __nv_bfloat16* X = static_cast<const __nv_bfloat16*>(p.x);
  const __nv_bfloat16* wlo = W + (size_t)(hb * HD + i0 + g) * D;
  const __nv_bfloat16* whi = W + (size_t)(hb * HD + HD / 2 + i0 + g) * D;
  if (threadIdx.x < 8) inv_freq[threadIdx.x] = rope_inv_freq(i0 + threadIdx.x, HD, p.theta);

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

  const int nkb = (D + 31) / 32;
  for (int kb0 = warp; kb0 < nkb; kb0 += WARPS * U) {
    uint4 wa[U], wb[U], xv[U][NT];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      // straight-line loads (clamped addresses, zeroed after) so that all of
      // them can be in flight together
      const int k = (kb0 + u * WARPS) * 32 + 8 * tq;
      const bool ok = k < D;
      const int kc = ok ? k : 0;
      wa[u] = ldg_stream(wlo + kc);
      wb[u] = ldg_stream(whi + kc);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int tok = n * 8 + g;
        xv[u][n] = ldg_keep(X + (size_t)(tok < T ? tok : 0) * D + kc);
        if (!(ok && tok < T)) xv[u][n] = make_uint4(0, 0, 0, 0);
      }
      if (!ok) wa[u] = wb[u] = make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        mma16816(acc[n], wa[u].x, wb[u].x, wa[u].y, wb[u].y, xv[u][n].x, xv[u][n].y);   // elements 0-3
        mma16816(acc[n], wa[u].z, wb[u].z, wa[u].w, wb[u].w, xv[u][n].z, xv[u][n].w);   // elements 4-7
      }
    }
  }

  // accumulators: c0,c1 = (lo row g, tokens 8n+2tq, +1); c2,c3 = (hi row g, same tokens)
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    red[warp][g][n * 8 + 2 * tq] = acc[n][0];
    red[warp][g][n * 8 + 2 * tq + 1] = acc[n][1];
    red[warp][g + 8][n * 8 + 2 * tq] = acc[n][2];
    red[warp][g + 8][n * 8 + 2 * tq + 1] = acc[n][3];
  }
  __syncthreads();

  const bool is_q = hb < p.nh, is_k = !is_q && hb < p.nh + p.nkv;
  for (int e = threadIdx.x; e < 8 * T; e += WARPS * 32) {
    if (e >= 8 * TP) break;
    const int r = e & 7, tok = e >> 3;
    float lo = 0.f, hi = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      lo += red[w][r][tok];
      hi += red[w][r + 8][tok];
    }
    const int b = tok / p.S, s = tok - b * p.S;
    const int pos = p.pos[tok];
    if (is_q || is_k) {
      float c, sn;
      rope_cos_sin(pos, inv_freq[r], &c, &sn);
      const float nl = lo * c - hi * sn, nh_ = hi * c + lo * sn;
      lo = nl;
      hi = nh_;
    }
    __nv_bfloat16* dst;
    if (is_q) {
      dst = static_cast<__nv_bfloat16*>(p.q_out) + (((size_t)b * p.nh + hb) * p.S + s) * HD;
    } else {
      if (pos < 0 || pos >= p.cap) {
        raise_error(p.err, GQA_DEVERR_POSITION_RANGE);
        continue;
      }
      const int jh = is_k ? hb - p.nh : hb - p.nh - p.nkv;
      dst = static_cast<__nv_bfloat16*>(is_k ? p.k_cache : p.v_cache) + (((size_t)b * p.nkv + jh) * p.cap + pos) * HD;
    }
    dst[i0 + r] = __float2bfloat16_rn(lo);
    dst[HD / 2 + i0 + r] = __float2bfloat16_rn(hi);
  }
}

template <int NT>
cudaError_t launch_nt(const QkvParams& p, cudaStream_t st) {
  const int N = (p.nh + 2 * p.nkv) * p.hd;
  const unsigned grid = (unsigned)(N / 16);
  switch (p.hd) {
    case 32: qkv_smallm_kernel<NT, 32><<<grid, WARPS * 32, 0, st>>>(p); break;
    case 64: qkv_smallm_kernel<NT, 64><<<grid, WARPS * 32, 0, st>>>(p); break;
    case 128: qkv_smallm_kernel<NT, 128><<<grid, WARPS * 32, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qkv_smallm(const QkvParams& p, cudaStream_t st) {
  const int T = p.B * p.S;
  if (T <= 8) return launch_nt<1>(p, st);
  if (T <= 16) return launch_nt<2>(p, st);
  if (T <= 32) return launch_nt<4>(p, st);
  if (T <= 64) return launch_nt<8>(p, st);
  return cudaErrorInvalidValue;
}

}  // namespace gqa
