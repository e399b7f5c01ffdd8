// Split-KV decode attention (steps a5-a6, bf16, head_dim 64 or 128).
//
// Decode reads each cached K/V row once per new token and does g
// multiply-adds per byte: it is HBM-bound (MHA -> GQA blog, sections
// 3.1-3.2).  The g query heads that share a KV head are stacked as the rows
// of tensor-core tiles, so one pass over a K/V row serves all of them and
// GQA's arithmetic intensity ~g is actually used.  tcgen05 wants M >= 64; for
// g <= 16 that would multiply the tensor work 4-16x for nothing, and this
// kernel's tensor work is far below the tensor roofline anyway, so it uses
// mma.sync m16n8k16 with 16 heads as M (g > 16: several head groups, each
// reading the K/V rows, the second time mostly from L2).
//
// CTA = (sequence b, KV head j, key split c, group of <= 16 heads).
// 5 warps:
//   warp 4     TMA producer: 64-key K and V tiles (128-byte swizzle, so the
//              ldmatrix reads below are conflict free) into a 3-4 stage ring
//   warps 0-3  each takes 16 keys of every tile: S = Q K^T (Q fragments
//              from a swizzled shared copy), mask keys past the split, online
//              softmax in log2 units, P kept in registers as the A fragment
//              of O += P V (V through ldmatrix.trans, shared by the MT tiles).
//              V rows past the valid keys are zeroed first, so NaN padding
//              never meets a zero P.
// The 4 warps' (m, l, O) are merged through shared memory.  A sequence with a
// single split writes its output directly.  Splits are then merged
// (log-sum-exp) in one of two ways:
//   cluster mode (the library picks the split, <= 8 per group): the splits of
//     a (b, j, head group) are one thread-block cluster; each sequence's
//     64-key tiles are dealt out evenly over its CTAs, and the CTAs read one
//     another's partials from distributed shared memory -- no workspace round
//     trip, which is what a small decode step's latency is made of;
//   workspace mode (fixed kv_split keys per split, or longer caches): every
//     split writes a partial (o unnormalised, m, l) to the workspace, bumps a
//     per-(b, j, head group) counter, and the last one to finish merges all
//     partials and resets the counter to zero.
#include "kernels.h"
#include "tc.cuh"

namespace gqa {
namespace {

constexpr int KT = 64;          // keys per tile
constexpr int kMaxClusterSplits = 8;  // portable cluster size
constexpr int THREADS = 160;    // 4 consumer warps + 1 producer warp

template <int HD, int MT>
struct DCfg {
  static constexpr int STAGES = HD == 128 ? 3 : 4;
  static constexpr int NBOX = HD / 64;
  static constexpr int BOX_BYTES = KT * 128;               // 64 rows x 128 bytes
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;      // one K or V tile
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int ROWS = 16 * MT;                     // head rows per CTA
  static constexpr int RED_STRIDE = HD + 4;                // fp32 merge rows
  static constexpr int RED_BYTES = 4 * ROWS * RED_STRIDE * 4;
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES > RED_BYTES ? STAGES * STAGE_BYTES : RED_BYTES;
  static constexpr int Q_BYTES = NBOX * ROWS * 128;        // swizzled bf16 Q rows
  static constexpr int SMEM = RING_BYTES + Q_BYTES + 2048 /*barriers*/ + 1024 /*align*/;
  // the final merge keeps (m, l) of every (head row, split) pair in the ring
  static_assert(ROWS * kMaxSplits * 8 <= RING_BYTES, "split merge does not fit in shared memory");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte offset of element (row, col) in a tile of 64-column boxes of `rows`
// 128-byte rows, 16-byte chunk c of a row stored at chunk c ^ (row & 7)
template <int ROWS_PER_BOX>
__device__ __forceinline__ uint32_t swz(int row, int col) {
  return (uint32_t)((col >> 6) * (ROWS_PER_BOX * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4));
}

template <int MT>
struct Bars {
  uint64_t full[4], empty[4];
  float ml[4][16 * MT][2];   // per warp, per head row: max, sum
  float cm[16 * MT][2];      // per head row: merged max, sum (or 1/sum)
  int last;
};

template <int HD, int MT, bool CL>
__global__ void __launch_bounds__(THREADS)
decode_mma_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                  DecodeParams p, int n_hgrp) {
  using C = DCfg<HD, MT>;
  constexpr int ROWS = C::ROWS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = smem + C::RING_BYTES;
  Bars<MT>* bars = reinterpret_cast<Bars<MT>*>(sq + C::Q_BYTES);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = blockIdx.z, j = blockIdx.y;
  // cluster mode: the n_split CTAs of one (sequence, KV head, head group)
  // are consecutive in x and form one cluster
  const int split = CL ? blockIdx.x % p.n_split : blockIdx.x / n_hgrp;
  const int hg = CL ? blockIdx.x / p.n_split : blockIdx.x % n_hgrp;
  const int g = p.nh / p.nkv;
  int* err = p.err;
  pdl_launch_dependents();
  pdl_wait();   // q, the lengths and the new cache rows may come from the kernel before this one

  int kv_len = p.kv_lens[b];
  if (kv_len > p.cap || kv_len < 0) {
    if (threadIdx.x == 0 && split == 0 && hg == 0) raise_error(err, GQA_DEVERR_KVLEN_RANGE);
    kv_len = kv_len > p.cap ? p.cap : 0;
  }
  const int h0 = j * g + hg * ROWS;
  const int rows = min(ROWS, g - hg * ROWS);
  int k_lo, k_hi, n_t;
  if (CL) {
    // the sequence's 64-key tiles dealt out evenly over the cluster; a CTA
    // may get none and still takes part in the merge
    const int tiles = (kv_len + KT - 1) / KT;
    const int t_lo = split * tiles / p.n_split, t_hi = (split + 1) * tiles / p.n_split;
    k_lo = t_lo * KT;
    k_hi = min(kv_len, t_hi * KT);
    n_t = t_hi - t_lo;
  } else {
    k_lo = split * p.split;
    if (k_lo >= kv_len) {  // no key of this sequence in this split (whole block)
      if (split == 0) {    // no key at all: the output rows are zero
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + ((size_t)b * p.nh + h0) * HD;
        for (int e = threadIdx.x; e < rows * HD; e += blockDim.x) out[e] = __float2bfloat16_rn(0.f);
      }
      return;
    }
    k_hi = min(kv_len, k_lo + p.split);
    n_t = (k_hi - k_lo + KT - 1) / KT;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 4);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      tc::prefetch_tmap(&tmk);
      tc::prefetch_tmap(&tmv);
      // cache row of a tile's first key: contiguous [B, nkv, cap, hd], or through
      // the block table (a 64-key tile never crosses a page: pages are
      // multiples of 64 keys and tiles start at multiples of 64); the table
      // entry is re-read only when the page changes
      int cur_page = -1, page_base = 0;
      auto tile_row = [&](int key) {
        if (!p.block_table) return (b * p.nkv + j) * p.cap + key;
        const int lp = key / p.page_size;
        if (lp != cur_page) {
          cur_page = lp;
          const int pg = __ldg(p.block_table + (size_t)b * p.max_pages + lp);
          if (pg < 0 || pg >= p.num_pages) {
            raise_error(err, GQA_DEVERR_PAGE_RANGE);
            page_base = p.num_pages * p.nkv * p.page_size;   // past the end: the copy reads zeros
          } else {
            page_base = (pg * p.nkv + j) * p.page_size;
          }
        }
        return page_base + (key - cur_page * p.page_size);
      };
      for (int t = 0; t < n_t; ++t) {
        const int s = t % C::STAGES;
        const int row = tile_row(k_lo + t * KT);
        if (!mbar_wait(&bars->empty[s], ((t / C::STAGES) & 1) ^ 1, err)) break;
        mbar_arrive_expect_tx(&bars->full[s], C::STAGE_BYTES);
        uint8_t* kt = smem + s * C::STAGE_BYTES;
        for (int bx = 0; bx < C::NBOX; ++bx) {
          tc::tma_load_2d(kt + bx * C::BOX_BYTES, &tmk, bx * 64, row, &bars->full[s]);
          tc::tma_load_2d(kt + C::TILE_BYTES + bx * C::BOX_BYTES, &tmv, bx * 64, row, &bars->full[s]);
        }
      }
      // every issued load has landed before the block may exit
      for (int t = max(0, n_t - C::STAGES); t < n_t; ++t)
        mbar_wait(&bars->full[t % C::STAGES], (t / C::STAGES) & 1, err);
    }
    __syncwarp();
    if (CL && p.n_split > 1) {  // the producer warp joins the two cluster barriers of the merge
      tc::cluster_sync();
      tc::cluster_sync();
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  // Q rows of this head group -> swizzled shared copy (zero rows past
  // `rows`), while the first K/V tiles are in flight.  All loads are issued
  // before the first store.
  {
    constexpr int QV = ROWS * (HD / 8) / 128;  // 16-byte vectors per consumer thread
    uint4 v[QV];
#pragma unroll
    for (int i = 0; i < QV; ++i) {
      const int e = threadIdx.x + i * 128, r = e / (HD / 8), c8 = (e % (HD / 8)) * 8;
      v[i] = make_uint4(0, 0, 0, 0);
      if (r < rows)
        v[i] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) +
                                               ((size_t)b * p.nh + h0 + r) * HD + c8);
    }
#pragma unroll
    for (int i = 0; i < QV; ++i) {
      const int e = threadIdx.x + i * 128, r = e / (HD / 8), c8 = (e % (HD / 8)) * 8;
      *reinterpret_cast<uint4*>(sq + swz<ROWS>(r, c8)) = v[i];
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
  }
  const int gr = lane >> 2, tq = lane & 3;  // fragment row group / thread in quad
  const int mrow = lane & 7, mat = lane >> 3;  // ldmatrix: row within matrix, matrix index
  const uint32_t q_base = smem_u32(sq);
  const float scale_log2 = 1.4426950408889634f * rsqrtf((float)HD);
  float m[MT][2], l[MT][2];
  float o[MT][HD / 8][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    m[mt][0] = m[mt][1] = -INFINITY;
    l[mt][0] = l[mt][1] = 0.f;
#pragma unroll
    for (int n = 0; n < HD / 8; ++n) o[mt][n][0] = o[mt][n][1] = o[mt][n][2] = o[mt][n][3] = 0.f;
  }

  for (int t = 0; t < n_t; ++t) {
    const int s = t % C::STAGES;
    const bool ok = mbar_wait(&bars->full[s], (t / C::STAGES) & 1, err);
    if (!__all_sync(0xffffffffu, ok)) break;
    const uint32_t kbase = smem_u32(smem + s * C::STAGE_BYTES);
    const uint32_t vbase = kbase + C::TILE_BYTES;
    const int slab = warp * 16;                         // first tile row of this warp
    const int nvalid = min(16, max(0, k_hi - (k_lo + t * KT + slab)));
    if (nvalid > 0) {
      if (nvalid < 16) {
        // zero V rows [nvalid, 16) of this warp's slab (whole 128-byte rows)
        for (int e = lane; e < (16 - nvalid) * 8 * C::NBOX; e += 32) {
          const int r = slab + nvalid + e / (8 * C::NBOX);
          const int rem = e % (8 * C::NBOX);
          tc::st_shared_v4(vbase + (rem / 8) * C::BOX_BYTES + r * 128 + (rem % 8) * 16, 0u, 0u, 0u, 0u);
        }
        tc::fence_proxy_async_smem();  // ordered before the next TMA write into this stage
        __syncwarp();
      }
      float sc[MT][2][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) sc[mt][nt][0] = sc[mt][nt][1] = sc[mt][nt][2] = sc[mt][nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks) {
        // K matrices: (keys 0-7, k lo), (keys 0-7, k hi), (keys 8-15, k lo), (keys 8-15, k hi)
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbase + swz<KT>(slab + (mat >> 1) * 8 + mrow, ks * 16 + (mat & 1) * 8), b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          // Q matrices: (rows 0-7, k lo), (rows 8-15, k lo), (rows 0-7, k hi), (rows 8-15, k hi)
          uint32_t qa[4];
          ldsm_x4(q_base + swz<ROWS>(mt * 16 + (mat & 1) * 8 + mrow, ks * 16 + (mat >> 1) * 8), qa[0], qa[1], qa[2],
                  qa[3]);
          mma16816(sc[mt][0], qa, b0, b1);
          mma16816(sc[mt][1], qa, b2, b3);
        }
      }
      uint32_t pa[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        // scale to log2 units and mask keys past the valid range
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = nt * 8 + 2 * tq + (e & 1);
            const float v = key < nvalid ? sc[mt][nt][e] * scale_log2 : -INFINITY;
            sc[mt][nt][e] = v;
            if (e < 2) mx0 = fmaxf(mx0, v); else mx1 = fmaxf(mx1, v);
          }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m[mt][0], mx0), mn1 = fmaxf(m[mt][1], mx1);  // finite: key 0 of the slab is valid
        const float al0 = tc::ex2(m[mt][0] - mn0), al1 = tc::ex2(m[mt][1] - mn1);
        m[mt][0] = mn0;
        m[mt][1] = mn1;
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          sc[mt][nt][0] = tc::ex2(sc[mt][nt][0] - mn0);
          sc[mt][nt][1] = tc::ex2(sc[mt][nt][1] - mn0);
          sc[mt][nt][2] = tc::ex2(sc[mt][nt][2] - mn1);
          sc[mt][nt][3] = tc::ex2(sc[mt][nt][3] - mn1);
          s0 += sc[mt][nt][0] + sc[mt][nt][1];
          s1 += sc[mt][nt][2] + sc[mt][nt][3];
        }
        s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
        s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
        l[mt][0] = l[mt][0] * al0 + s0;
        l[mt][1] = l[mt][1] * al1 + s1;
#pragma unroll
        for (int n = 0; n < HD / 8; ++n) {
          o[mt][n][0] *= al0;
          o[mt][n][1] *= al0;
          o[mt][n][2] *= al1;
          o[mt][n][3] *= al1;
        }
        pa[mt][0] = pack_bf16x2(sc[mt][0][0], sc[mt][0][1]);
        pa[mt][1] = pack_bf16x2(sc[mt][0][2], sc[mt][0][3]);
        pa[mt][2] = pack_bf16x2(sc[mt][1][0], sc[mt][1][1]);
        pa[mt][3] = pack_bf16x2(sc[mt][1][2], sc[mt][1][3]);
      }
#pragma unroll
      for (int np = 0; np < HD / 16; ++np) {
        // V matrices: (keys 0-7, cols 0-7), (keys 8-15, cols 0-7), (keys 0-7, cols 8-15), (keys 8-15, cols 8-15)
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbase + swz<KT>(slab + (mat & 1) * 8 + mrow, np * 16 + (mat >> 1) * 8), b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          mma16816(o[mt][2 * np], pa[mt], b0, b1);
          mma16816(o[mt][2 * np + 1], pa[mt], b2, b3);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->empty[s]);
  }

  // ------------------------------------------------------------------ merge the 4 warps
  if (tq == 0) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      bars->ml[warp][mt * 16 + gr][0] = m[mt][0];
      bars->ml[warp][mt * 16 + gr][1] = l[mt][0];
      bars->ml[warp][mt * 16 + gr + 8][0] = m[mt][1];
      bars->ml[warp][mt * 16 + gr + 8][1] = l[mt][1];
    }
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");   // consumers only; the ring is idle now
  float* red = reinterpret_cast<float*>(smem);
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      M0 = fmaxf(M0, bars->ml[w][mt * 16 + gr][0]);
      M1 = fmaxf(M1, bars->ml[w][mt * 16 + gr + 8][0]);
    }
    const float f0 = m[mt][0] == -INFINITY ? 0.f : tc::ex2(m[mt][0] - M0);
    const float f1 = m[mt][1] == -INFINITY ? 0.f : tc::ex2(m[mt][1] - M1);
#pragma unroll
    for (int n = 0; n < HD / 8; ++n) {
      const int c = n * 8 + 2 * tq;
      float* r0 = red + (warp * ROWS + mt * 16 + gr) * C::RED_STRIDE + c;
      float* r1 = r0 + 8 * C::RED_STRIDE;
      r0[0] = o[mt][n][0] * f0;
      r0[1] = o[mt][n][1] * f0;
      r1[0] = o[mt][n][2] * f1;
      r1[1] = o[mt][n][3] * f1;
    }
  }
  const int tid = threadIdx.x;
  if (tid < ROWS) {  // this CTA's max and sum per head row, over its 4 warps
    float M = -INFINITY, L = 0.f;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, bars->ml[w][tid][0]);
    for (int w = 0; w < 4; ++w) {
      const float mw = bars->ml[w][tid][0];
      if (mw != -INFINITY) L += bars->ml[w][tid][1] * tc::ex2(mw - M);
    }
    bars->cm[tid][0] = M;
    bars->cm[tid][1] = L;
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  auto red_sum = [&](int r, int c) {
    return red[(0 * ROWS + r) * C::RED_STRIDE + c] + red[(1 * ROWS + r) * C::RED_STRIDE + c] +
           red[(2 * ROWS + r) * C::RED_STRIDE + c] + red[(3 * ROWS + r) * C::RED_STRIDE + c];
  };
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  if (CL && p.n_split > 1) {
    // ---------------------------------------------------------- cluster merge
    // this CTA's o (summed over its 4 warps, relative to its max) in place of
    // warp 0's rows; (max, sum) per row are in bars->cm
    for (int e = tid; e < rows * HD; e += 128) {
      const int r = e / HD, c = e % HD;
      red[r * C::RED_STRIDE + c] = red_sum(r, c);
    }
    tc::cluster_sync();
    // float4 output pieces dealt out over the cluster's consumer threads; each
    // reads the n_split partial rows from the CTAs' shared memory
    const int nsp = p.n_split;
    const uint32_t red_u = smem_u32(red), cm_u = smem_u32(&bars->cm[0][0]);
    for (int e = split * 128 + tid; e < rows * (HD / 4); e += nsp * 128) {
      const int r = e / (HD / 4), c = (e % (HD / 4)) * 4;
      float2 ml[8];
      float M = -INFINITY;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q < nsp) {
          ml[q] = tc::ld_dsmem_f32x2(tc::mapa_shared(cm_u + r * 8, q));
          M = fmaxf(M, ml[q].x);
        }
      }
      float L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q < nsp && ml[q].x != -INFINITY) {
          const float w = tc::ex2(ml[q].x - M);
          const float4 v = tc::ld_dsmem_f32x4(tc::mapa_shared(red_u + (r * C::RED_STRIDE + c) * 4, q));
          L += ml[q].y * w;
          acc.x = fmaf(v.x, w, acc.x);
          acc.y = fmaf(v.y, w, acc.y);
          acc.z = fmaf(v.z, w, acc.z);
          acc.w = fmaf(v.w, w, acc.w);
        }
      }
      const float inv = L > 0.f ? 1.f / L : 0.f;
      __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(out + ((size_t)b * p.nh + h0 + r) * HD + c);
      dst[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
      dst[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    }
    tc::cluster_sync();  // no CTA leaves while another may still read its shared memory
    return;
  }
  const int n_active = CL ? 1 : (kv_len + p.split - 1) / p.split;   // splits that hold keys of this sequence
  if (n_active == 1) {
    // the only split: normalise and write the output directly
    for (int e = tid; e < rows * HD; e += 128) {
      const int r = e / HD, c = e % HD;
      const float L = bars->cm[r][1];
      out[((size_t)b * p.nh + h0 + r) * HD + c] = __float2bfloat16_rn(L > 0.f ? red_sum(r, c) / L : 0.f);
    }
    return;
  }
  // write this split's partial (o unnormalised, m in log2 units, l)
  for (int e = tid; e < rows * HD; e += 128) {
    const int r = e / HD, c = e % HD;
    float* row = p.ws + (((size_t)b * p.nh + h0 + r) * p.n_split + split) * (HD + kWsPad);
    row[c] = red_sum(r, c);
    if (c == 0) {
      row[HD] = bars->cm[r][0];
      row[HD + 1] = bars->cm[r][1];
    }
  }
  // the last split of this (sequence, KV head, head group) to finish merges them all
  __threadfence();
  asm volatile("bar.sync 1, 128;" ::: "memory");
  unsigned* counter = p.counters + ((size_t)b * p.nkv + j) * n_hgrp + hg;
  if (tid == 0) bars->last = atomicAdd(counter, 1u) == (unsigned)(n_active - 1);
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (!bars->last) return;
  __threadfence();
  // merge: (1) every (head row, split) pair's (m, l) is fetched at once into
  // shared memory (one round trip); (2) per head row, lanes over the splits
  // -> max, sum and one weight 2^(m_s - M) / L per split, from shared memory
  // only; (3) every thread takes float4 output columns and sums the splits
  // with independent loads.
  const size_t stride = HD + kWsPad;
  float2* mls = reinterpret_cast<float2*>(red);  // [rows][n_active]: (m, l), then (weight, -)
  for (int e = tid; e < rows * n_active; e += 128) {
    const int r = e / n_active, s = e - r * n_active;
    mls[e] = __ldcg(reinterpret_cast<const float2*>(p.ws + (((size_t)b * p.nh + h0 + r) * p.n_split + s) * stride + HD));
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  for (int r = warp; r < rows; r += 4) {
    float2* ml = mls + r * n_active;
    float M = -INFINITY;
    for (int s = lane; s < n_active; s += 32) M = fmaxf(M, ml[s].x);
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
    float L = 0.f;
    for (int s = lane; s < n_active; s += 32) {
      const float2 v = ml[s];
      const float e = v.x == -INFINITY ? 0.f : tc::ex2(v.x - M);
      ml[s].x = e;
      L += v.y * e;
    }
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o2);
    const float inv = L > 0.f ? 1.f / L : 0.f;
    for (int s = lane; s < n_active; s += 32) ml[s].x *= inv;
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  for (int e = tid; e < rows * (HD / 4); e += 128) {
    const int r = e / (HD / 4), c = (e % (HD / 4)) * 4;
    const float* part = p.ws + ((size_t)b * p.nh + h0 + r) * p.n_split * stride + c;
    const float2* w = mls + r * n_active;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int s = 0; s < n_active; ++s) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(part + s * stride));
      const float ws_ = w[s].x;
      acc.x = fmaf(v.x, ws_, acc.x);
      acc.y = fmaf(v.y, ws_, acc.y);
      acc.z = fmaf(v.z, ws_, acc.z);
      acc.w = fmaf(v.w, ws_, acc.w);
    }
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(out + ((size_t)b * p.nh + h0 + r) * HD + c);
    dst[0] = __floats2bfloat162_rn(acc.x, acc.y);
    dst[1] = __floats2bfloat162_rn(acc.z, acc.w);
  }
  if (tid == 0) atomicExch(counter, 0u);  // leave the counter at zero for the next call
}

template <int HD, int MT, bool CL>
cudaError_t launch_hd(const DecodeParams& p, cudaStream_t st) {
  using C = DCfg<HD, MT>;
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = smem_attr_once(attr_set, reinterpret_cast<const void*>(decode_mma_kernel<HD, MT, CL>), C::SMEM);
      e != cudaSuccess)
    return e;
  CUtensorMap tk, tv;
  const uint64_t rows = p.block_table ? (uint64_t)p.num_pages * p.nkv * p.page_size : (uint64_t)p.B * p.nkv * p.cap;
  if (!make_tmap_bf16_2d(&tk, p.k_cache, HD, rows, HD * 2, 64, KT)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tv, p.v_cache, HD, rows, HD * 2, 64, KT)) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)(p.n_split * p.n_hgrp), p.nkv, p.B);
  if (!CL) return launch_ex(decode_mma_kernel<HD, MT, false>, grid, dim3(THREADS), C::SMEM, st, 1u, tk, tv, p, p.n_hgrp);
  return launch_ex(decode_mma_kernel<HD, MT, true>, grid, dim3(THREADS), C::SMEM, st, (unsigned)p.n_split, tk, tv, p,
                   p.n_hgrp);
}

// Splits per (sequence, KV head, head group) for the cluster-merged decode,
// or 0 to use the workspace splits: about two CTAs per SM over the whole
// problem and at most 2048 keys a CTA, within one portable cluster (<= 8).
int cluster_splits(const DecodeParams& p) {
  const long long groups = (long long)p.B * p.nkv * p.n_hgrp;
  const int by_len = (p.cap + 2047) / 2048;
  if (by_len > kMaxClusterSplits) return 0;
  long long n = (2 * 148 + groups - 1) / groups;
  if (n < by_len) n = by_len;
  if (n > kMaxClusterSplits) n = kMaxClusterSplits;
  const int tiles = (p.cap + KT - 1) / KT;
  if (n > tiles) n = tiles;
  return (int)(n < 1 ? 1 : n);
}

}  // namespace

cudaError_t launch_decode_mma(const DecodeParams& p, cudaStream_t st) {
  switch (p.hd) {
    case 64: return p.cluster ? launch_hd<64, 1, true>(p, st) : launch_hd<64, 1, false>(p, st);
    case 128: return p.cluster ? launch_hd<128, 1, true>(p, st) : launch_hd<128, 1, false>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

int launch_decode(const DecodeParams& p0, bool bf16, cudaStream_t st, cudaError_t* err) {
  if (bf16 && p0.auto_split) {
    // large batches with large head groups: tcgen05 tiles (mma.sync would be
    // tensor-bound there), splits merged inside a cluster; contiguous or
    // paged (each 64-key tile mapped to its page)
    const int nc = decode_tc_splits(p0);
    if (nc > 0) {
      DecodeParams p = p0;
      p.cluster = 1;
      p.n_split = nc;
      *err = launch_decode_tc(p, st);
      return 1;
    }
  }
  if (bf16 && decode_hn_ok(p0.B, p0.nh, p0.nkv, p0.hd, p0.cap, p0.auto_split != 0)) {
    // the other large problems with head groups of 17..64 (caches past the
    // cluster kernel's 8 x 2048 keys): keys as the tcgen05 rows, equal key
    // ranges per SM.  On the B 64 MQA workload the cluster kernel above
    // measured 42 us back to back against this kernel's 51 us, contiguous or
    // with 64-key pages.
    *err = launch_decode_hn(p0, st);
    return 1;
  }
  if (bf16 && (p0.hd == 64 || p0.hd == 128)) {  // merges its splits itself
    DecodeParams p = p0;
    const int nc = p.auto_split ? cluster_splits(p) : 0;
    if (nc > 0) {
      p.cluster = 1;
      p.n_split = nc;
    }
    *err = launch_decode_mma(p, st);
    return 1;
  }
  cudaError_t e = launch_decode_simt(p0, bf16, st);
  if (e == cudaSuccess) e = launch_decode_combine(p0, bf16, st);
  *err = e;
  return 2;
}

}  // namespace gqa
