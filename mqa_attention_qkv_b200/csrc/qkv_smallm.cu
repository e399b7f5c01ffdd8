// Fused QKV projection for a handful of tokens (T <= 64: the one-token decode
// steps of a generation loop), with the same RoPE + head-major scatter
// epilogue as the big tensor-core GEMM (steps a1-a3, bf16).
//
// With T tokens of hidden size D the projection reads the whole W_qkv
// (N x D) to do 2*T*N*D flops: it is bound by the W stream (the "batch-1 is
// matrix-vector, memory-bound" case of the MHA -> GQA blog, section 3.1), so
// the design goal is to spread W over every SM with many bytes in flight.
// Both kernels below work in units of 16 rows of W (8 RoPE pairs, see the
// register kernel); the TMA-ring kernel (further down) serves hidden % 64 == 0
// when the tokens' hidden states fit in shared memory, the register kernel
// everything else.
//
// Register kernel.  CTA = 16 rows of W: 8 consecutive features at offset i0 of the first half
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
#include <atomic>

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

// Epilogue of one RoPE pair: features i0 + r (lo) and hd/2 + i0 + r (hi) of
// head block hb for token tok.  Q and K heads are rotated by the token's
// position (rotate-half form), then Q goes to [B, nh, S, hd] and K/V to
// cache row `pos` of [B, nkv, cap, hd]; a position outside the cache is
// flagged and skipped.
template <int HD>
__device__ __forceinline__ void rope_store_pair(const QkvParams& p, int hb, int i0, int r, int tok, float lo,
                                                float hi, double inv_freq) {
  const bool is_q = hb < p.nh, is_k = !is_q && hb < p.nh + p.nkv;
  const int b = tok / p.S, s = tok - b * p.S;
  const int pos = p.pos[tok];
  if (is_q || is_k) {
    float c, sn;
    rope_cos_sin(pos, inv_freq, &c, &sn);
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
      return;
    }
    const int jh = is_k ? hb - p.nh : hb - p.nh - p.nkv;
    dst = static_cast<__nv_bfloat16*>(is_k ? p.k_cache : p.v_cache) + (((size_t)b * p.nkv + jh) * p.cap + pos) * HD;
  }
  dst[i0 + r] = __float2bfloat16_rn(lo);
  dst[HD / 2 + i0 + r] = __float2bfloat16_rn(hi);
}

template <int NT, int HD>
__global__ void __launch_bounds__(WARPS * 32, 2) qkv_smallm_kernel(QkvParams p) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
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

  for (int e = threadIdx.x; e < 8 * T; e += WARPS * 32) {
    if (e >= 8 * TP) break;
    const int r = e & 7, tok = e >> 3;
    float lo = 0.f, hi = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      lo += red[w][r][tok];
      hi += red[w][r + 8][tok];
    }
    rope_store_pair<HD>(p, hb, i0, r, tok, lo, hi, inv_freq[r]);
  }
}

// ---------------------------------------------------------------------------
// Streaming variant, used when hidden % 64 == 0 and the tokens' hidden states
// fit in shared memory next to the W ring (the usual one-token step).  The
// register kernel above loads, waits and multiplies in rounds, and its 16-row
// CTAs come in more than one wave; here persistent CTAs (one per SM, or two
// with a shorter ring when the hidden states are small and there are more
// units than SMs) walk the same 16-row work units u = blockIdx.x,
// +gridDim.x, ...  and a TMA producer warp keeps a ring of W slabs in flight
// across unit boundaries, so the W stream does not drain between units or
// waves.
//
//   X   [T, hidden] -> shared memory once per CTA by the consumer threads, in
//       the layout of 64-column, 128-byte-swizzled boxes of TP rows (rows past
//       T zero), while the producer starts the W ring
//   W   per stage: the 8 lo rows and the 8 hi rows of the unit over 512
//       columns (two 3-D boxes of 8 column blocks x 8 rows x 64 columns)
//   consumer warp w takes column block w of every stage: ldmatrix fragments
//       of W (rows as M) and X (tokens as N), mma.sync m16n8k16
//   after a unit's last stage the 8 warps' sums meet in shared memory and the
//   RoPE + scatter epilogue of the register kernel runs (frequencies from a
//   per-CTA table).  Measured on B200, handing the epilogue to a warp of its
//   own was slower: one warp's serial double-precision angle reductions then
//   form the kernel's tail.
constexpr int SW_WARPS = 8;                       // consumer warps (+1 producer)
constexpr int SW_STAGES = 6;                      // ring depth with one CTA per SM (at most)
constexpr int SW_KB = 8;                          // 64-column blocks per stage
constexpr int SW_HALF = SW_KB * 8 * 128;          // 8 rows x 512 columns
constexpr int SW_STAGE = 2 * SW_HALF;             // lo + hi rows
constexpr int SW_SMEM_MAX = 227 * 1024;
constexpr int SW_MAX_NBLK = 256;                  // column-block counts whose launch shape is cached
constexpr int HD_MAX = 128;
static_assert(SW_KB == SW_WARPS, "one column block per consumer warp and stage");

inline size_t stream_smem(int NT, int nblk, int stages = SW_STAGES) {
  const size_t TP = (size_t)NT * 8;
  return 1024 /*align*/ + (size_t)stages * SW_STAGE + (size_t)nblk * TP * 128 +
         (size_t)SW_WARPS * 16 * (TP + 1) * 4 + 2 * SW_STAGES * 8 + (size_t)(HD_MAX / 2) * 8;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// Epilogues of the streaming kernel.  A work unit is 16 rows of W: 8 "lo"
// rows at unit_row(u) and 8 "hi" rows HD/2 further on (HD = 16: 16
// consecutive rows).  store() gets the finished dot products of lo row
// unit_row(u) + r and its hi partner with token `tok`.
template <int HD_>
struct StreamQkv {                         // QKV projection: RoPE pair + scatter
  static constexpr int HD = HD_;
  using Params = QkvParams;
  __device__ static int T(const Params& p) { return p.B * p.S; }
  __device__ static int K(const Params& p) { return p.hidden; }
  __device__ static const void* X(const Params& p) { return p.x; }
  __device__ static int* err(const Params& p) { return p.err; }
  __device__ static void init(const Params& p, double* table) {
    for (int f = threadIdx.x; f < HD / 2; f += SW_WARPS * 32) table[f] = rope_inv_freq(f, HD, p.theta);
  }
  __device__ static void store(const Params& p, int u, int r, int tok, float lo, float hi, const double* table) {
    constexpr int GROUPS = HD / 16;
    const int hb = u / GROUPS, i0 = (u % GROUPS) * 8;
    rope_store_pair<HD>(p, hb, i0, r, tok, lo, hi, table[i0 + r]);
  }
};

struct StreamResidual {                    // output projection: + residual, round once
  static constexpr int HD = 16;
  using Params = OprojParams;
  __device__ static int T(const Params& p) { return p.T; }
  __device__ static int K(const Params& p) { return p.K; }
  __device__ static const void* X(const Params& p) { return p.x; }
  __device__ static int* err(const Params& p) { return p.err; }
  __device__ static void init(const Params&, double*) {}
  __device__ static void store(const Params& p, int u, int r, int tok, float lo, float hi, const double*) {
    const size_t o = (size_t)tok * p.N + u * 16 + r;
    const __nv_bfloat16* res = static_cast<const __nv_bfloat16*>(p.residual);
    if (res) {
      lo += __bfloat162float(res[o]);
      hi += __bfloat162float(res[o + 8]);
    }
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    out[o] = __float2bfloat16_rn(lo);
    out[o + 8] = __float2bfloat16_rn(hi);
  }
};

template <int NT, class Epi>
__global__ void __launch_bounds__((SW_WARPS + 1) * 32, 1)
w_stream_kernel(const __grid_constant__ CUtensorMap tmw, typename Epi::Params p,
                int n_units, int nstages) {
  constexpr int TP = NT * 8;
  constexpr int HD = Epi::HD;
  constexpr int GROUPS = HD / 16;
  constexpr int XBOX = TP * 128;                   // one 64-column block of X
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nblk = Epi::K(p) / 64;
  const int nst = (nblk + SW_KB - 1) / SW_KB;
  uint8_t* ring = smem;
  uint8_t* xs = smem + nstages * SW_STAGE;
  float* red = reinterpret_cast<float*>(xs + (size_t)nblk * XBOX);      // [warp][16 rows][TP + 1]
  uint64_t* full = reinterpret_cast<uint64_t*>(red + SW_WARPS * 16 * (TP + 1));
  uint64_t* empty = full + SW_STAGES;
  double* inv_freq = reinterpret_cast<double*>(empty + SW_STAGES);   // [HD / 2]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int T = Epi::T(p);
  int* err = Epi::err(p);
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], SW_WARPS);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();   // the inputs may come from the kernel before this one

  if (warp == SW_WARPS) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tc::prefetch_tmap(&tmw);
      // ring slot s and its phase parity, advanced without a division (the
      // ring depth is a launch parameter; a runtime divide per stage
      // measured as a several-microsecond loss)
      int it = 0, s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int rlo = (u / GROUPS) * HD + (u % GROUPS) * 8;
        for (int st = 0; st < nst; ++st) {
          if (!mbar_wait(&empty[s], ph ^ 1, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], SW_STAGE);
          tc::tma_load_3d(ring + s * SW_STAGE, &tmw, 0, rlo, st * SW_KB, &full[s]);
          tc::tma_load_3d(ring + s * SW_STAGE + SW_HALF, &tmw, 0, rlo + HD / 2, st * SW_KB, &full[s]);
          ++it;
          if (++s == nstages) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      // every issued copy has landed before the block may exit: walk back
      // over the last min(it, nstages) copies
      for (int k = 0; k < min(it, nstages); ++k) {
        if (--s < 0) {
          s = nstages - 1;
          ph ^= 1;
        }
        mbar_wait(&full[s], ph, err);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int g = lane >> 2, tq = lane & 3;
  const int mrow = lane & 7, mat = lane >> 3;     // ldmatrix: row in matrix, matrix index
  const uint32_t ring_u = smem_u32(ring), xs_u = smem_u32(xs);
  {
    // X -> shared memory (the swizzled layout of a 64-column TMA box of TP
    // rows; rows past T zero) by the consumer threads, 8 vectors in flight
    // each, while the producer fills the W ring.  (Fetched by TMA next to
    // the W slabs, the same X measured markedly slower on B200.)
    const __nv_bfloat16* X = static_cast<const __nv_bfloat16*>(Epi::X(p));
    const int hidden = Epi::K(p);
    const int nchunk = nblk * TP * 8;
    for (int e0 = threadIdx.x; e0 < nchunk; e0 += SW_WARPS * 32 * 8) {
      uint4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i * SW_WARPS * 32;
        const int kb = e / (TP * 8), rem = e % (TP * 8), row = rem / 8, ch = rem % 8;
        v[i] = make_uint4(0, 0, 0, 0);
        if (e < nchunk && row < T)
          v[i] = *reinterpret_cast<const uint4*>(X + (size_t)row * hidden + kb * 64 + ch * 8);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i * SW_WARPS * 32;
        const int kb = e / (TP * 8), rem = e % (TP * 8), row = rem / 8, ch = rem % 8;
        if (e < nchunk) *reinterpret_cast<uint4*>(xs + kb * XBOX + row * 128 + ((ch ^ (row & 7)) << 4)) = v[i];
      }
    }
    // the epilogue's per-CTA table (the RoPE frequencies of the head dimension)
    Epi::init(p, inv_freq);
    asm volatile("bar.sync 1, %0;" ::"n"(SW_WARPS * 32) : "memory");
  }
  bool dead = false;
  int s = 0;            // ring slot and phase parity, advanced as in the producer
  uint32_t ph = 0;
  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    for (int st = 0; st < nst; ++st) {
      if (!dead) dead = !__all_sync(0xffffffffu, mbar_wait(&full[s], ph, err));
      const int kb = st * SW_KB + warp;
      if (!dead && kb < nblk) {
        const uint32_t wb = ring_u + s * SW_STAGE + warp * 1024;
        const uint32_t xb = xs_u + kb * XBOX;
        if (NT == 1) {
#pragma unroll
          for (int ks = 0; ks < 4; ks += 2) {
            // X matrices: (tokens 0-7, 16-byte chunks 2ks .. 2ks+3): k16 steps ks and ks + 1
            uint32_t b0, b1, b2, b3;
            ldsm_x4(xb + mrow * 128 + (((2 * ks + mat) ^ mrow) << 4), b0, b1, b2, b3);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // W matrices: (lo rows, k 0-7), (hi rows, k 0-7), (lo, k 8-15), (hi, k 8-15)
              uint32_t a0, a1, a2, a3;
              const int wch = 2 * (ks + h) + (mat >> 1);
              ldsm_x4(wb + (mat & 1) * SW_HALF + mrow * 128 + ((wch ^ mrow) << 4), a0, a1, a2, a3);
              mma16816(acc[0], a0, a1, a2, a3, h ? b2 : b0, h ? b3 : b1);
            }
          }
        } else {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            // W matrices: (lo rows, k 0-7), (hi rows, k 0-7), (lo, k 8-15), (hi, k 8-15)
            uint32_t a0, a1, a2, a3;
            const int wch = 2 * ks + (mat >> 1);
            ldsm_x4(wb + (mat & 1) * SW_HALF + mrow * 128 + ((wch ^ mrow) << 4), a0, a1, a2, a3);
#pragma unroll
            for (int np = 0; np < NT; np += 2) {
              // X matrices: (tokens np*8.., k 0-7), (same, k 8-15), (tokens (np+1)*8.., k 0-7), (same, k 8-15)
              const int tok = (np + (mat >> 1)) * 8 + mrow;
              const int xch = 2 * ks + (mat & 1);
              uint32_t b0, b1, b2, b3;
              ldsm_x4(xb + tok * 128 + ((xch ^ mrow) << 4), b0, b1, b2, b3);
              mma16816(acc[np], a0, a1, a2, a3, b0, b1);
              mma16816(acc[np + 1 < NT ? np + 1 : np], a0, a1, a2, a3, b2, b3);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0 && !dead) mbar_arrive(&empty[s]);
      if (++s == nstages) {
        s = 0;
        ph ^= 1;
      }
    }

    // the 8 warps' partial sums: c0,c1 = (lo row g, tokens 8n+2tq, +1); c2,c3 = (hi row g, same)
    float* rw = red + warp * 16 * (TP + 1);
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      rw[g * (TP + 1) + n * 8 + 2 * tq] = acc[n][0];
      rw[g * (TP + 1) + n * 8 + 2 * tq + 1] = acc[n][1];
      rw[(g + 8) * (TP + 1) + n * 8 + 2 * tq] = acc[n][2];
      rw[(g + 8) * (TP + 1) + n * 8 + 2 * tq + 1] = acc[n][3];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(SW_WARPS * 32) : "memory");
    for (int e = threadIdx.x; e < 8 * T; e += SW_WARPS * 32) {
      const int r = e & 7, tok = e >> 3;
      float lo = 0.f, hi = 0.f;
#pragma unroll
      for (int w = 0; w < SW_WARPS; ++w) {
        lo += red[(w * 16 + r) * (TP + 1) + tok];
        hi += red[(w * 16 + r + 8) * (TP + 1) + tok];
      }
      if (!dead) Epi::store(p, u, r, tok, lo, hi, inv_freq);
    }
    asm volatile("bar.sync 1, %0;" ::"n"(SW_WARPS * 32) : "memory");
  }
}

template <int NT, class Epi>
cudaError_t launch_stream_epi(const typename Epi::Params& p, const void* w, int K, int N, int num_sms,
                              cudaStream_t st) {
  const int nblk = K / 64;
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = smem_attr_once(attr_set, reinterpret_cast<const void*>(w_stream_kernel<NT, Epi>), SW_SMEM_MAX);
      e != cudaSuccess)
    return e;
  const int n_units = N / 16;
  // More units than SMs and small hidden states: two CTAs per SM with a
  // shorter ring each, so that a few hundred units run in one wave instead
  // of a few SMs taking a second unit after everyone else is done.
  int stages = SW_STAGES, per_sm = 1;
  if (n_units > num_sms) {
    // the deepest ring with which two CTAs fit on an SM (0: none), found once
    // per column-block count (a host-side occupancy query per call would sit
    // in the launch path of every generation step)
    static std::atomic<int> two_per_sm[SW_MAX_NBLK + 1];   // 0 unknown, -1 none, else stages
    int known = nblk <= SW_MAX_NBLK ? two_per_sm[nblk].load(std::memory_order_relaxed) : 0;
    if (known == 0) {
      known = -1;
      for (int s2 = SW_STAGES; s2 >= 3; --s2) {
        int fit = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fit, w_stream_kernel<NT, Epi>, (SW_WARPS + 1) * 32,
                                                          stream_smem(NT, nblk, s2)) != cudaSuccess) {
          cudaGetLastError();
          break;
        }
        if (fit >= 2) {
          known = s2;
          break;
        }
      }
      if (nblk <= SW_MAX_NBLK) two_per_sm[nblk].store(known, std::memory_order_relaxed);
    }
    if (known > 0) {
      stages = known;
      per_sm = 2;
    }
  }
  const size_t smem = stream_smem(NT, nblk, stages);
  CUtensorMap tw;
  // W viewed as [column block][row][64 columns]: a box is 8 blocks x 8 rows
  const uint64_t wd[3] = {64, (uint64_t)N, (uint64_t)nblk};
  const uint64_t ws[2] = {(uint64_t)K * 2, 128};
  const uint32_t wbox[3] = {64, 8, SW_KB};
  if (!make_tmap_bf16_3d(&tw, w, wd, ws, wbox)) return cudaErrorInvalidValue;
  const int grid = n_units < per_sm * num_sms ? n_units : per_sm * num_sms;
  return launch_ex(w_stream_kernel<NT, Epi>, dim3((unsigned)grid), dim3((SW_WARPS + 1) * 32), smem, st, 1u, tw, p,
                   n_units, stages);
}

template <int NT, int HD>
cudaError_t launch_stream_hd(const QkvParams& p, int num_sms, cudaStream_t st) {
  return launch_stream_epi<NT, StreamQkv<HD>>(p, p.w, p.hidden, (p.nh + 2 * p.nkv) * HD, num_sms, st);
}

template <int NT>
cudaError_t launch_stream(const QkvParams& p, int num_sms, cudaStream_t st) {
  switch (p.hd) {
    case 32: return launch_stream_hd<NT, 32>(p, num_sms, st);
    case 64: return launch_stream_hd<NT, 64>(p, num_sms, st);
    case 128: return launch_stream_hd<NT, 128>(p, num_sms, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int NT>
cudaError_t launch_nt(const QkvParams& p, cudaStream_t st) {
  const int N = (p.nh + 2 * p.nkv) * p.hd;
  const unsigned grid = (unsigned)(N / 16);
  switch (p.hd) {
    case 32: return launch_ex(qkv_smallm_kernel<NT, 32>, dim3(grid), dim3(WARPS * 32), 0, st, 1u, p);
    case 64: return launch_ex(qkv_smallm_kernel<NT, 64>, dim3(grid), dim3(WARPS * 32), 0, st, 1u, p);
    case 128: return launch_ex(qkv_smallm_kernel<NT, 128>, dim3(grid), dim3(WARPS * 32), 0, st, 1u, p);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool oproj_stream_fits(const OprojParams& p) {
  if (p.T > 64 || p.K % 64 != 0 || p.N % 16 != 0) return false;
  const int nt = p.T <= 8 ? 1 : p.T <= 16 ? 2 : p.T <= 32 ? 4 : 8;
  return stream_smem(nt, p.K / 64) <= (size_t)SW_SMEM_MAX;
}

cudaError_t launch_oproj_stream(const OprojParams& p, int num_sms, cudaStream_t st) {
  if (!oproj_stream_fits(p)) return cudaErrorInvalidValue;
  switch (p.T <= 8 ? 1 : p.T <= 16 ? 2 : p.T <= 32 ? 4 : 8) {
    case 1: return launch_stream_epi<1, StreamResidual>(p, p.w, p.K, p.N, num_sms, st);
    case 2: return launch_stream_epi<2, StreamResidual>(p, p.w, p.K, p.N, num_sms, st);
    case 4: return launch_stream_epi<4, StreamResidual>(p, p.w, p.K, p.N, num_sms, st);
    default: return launch_stream_epi<8, StreamResidual>(p, p.w, p.K, p.N, num_sms, st);
  }
}

cudaError_t launch_qkv_smallm(const QkvParams& p, int num_sms, cudaStream_t st) {
  const int T = p.B * p.S;
  const int nt = T <= 8 ? 1 : T <= 16 ? 2 : T <= 32 ? 4 : T <= 64 ? 8 : 0;
  if (nt == 0) return cudaErrorInvalidValue;
  if (p.hidden % 64 == 0 && stream_smem(nt, p.hidden / 64) <= (size_t)SW_SMEM_MAX) {
    switch (nt) {
      case 1: return launch_stream<1>(p, num_sms, st);
      case 2: return launch_stream<2>(p, num_sms, st);
      case 4: return launch_stream<4>(p, num_sms, st);
      default: return launch_stream<8>(p, num_sms, st);
    }
  }
  switch (nt) {
    case 1: return launch_nt<1>(p, st);
    case 2: return launch_nt<2>(p, st);
    case 4: return launch_nt<4>(p, st);
    default: return launch_nt<8>(p, st);
  }
}

}  // namespace gqa
