// Output projection with residual for a few tokens (T <= 64: the decode steps
// of a generation loop), bf16, on the Blackwell tensor cores.
//
// out[T, N] = attn[T, K] . W_o[N, K]^T + residual[T, N] (the custom-op
// overhead gist's LlamaAttention.forward ends in its output projection, and
// its decoder layer adds the residual stream).  With a handful of tokens the
// product reads all of W_o to do 2*T*N*K flops, so it is bound by the W_o
// stream (the matrix-vector case of the MHA -> GQA blog, section 3.1); the
// design spreads W_o over as many SMs as possible with many bytes in flight.
//
// "Swap AB": W_o rows are the MMA's M = 128 and the tokens its N (T padded to
// NT = 16, 32 or 64), so a tile wastes nothing on padding rows of W.  A
// 128-row block of W_o alone would keep only N / 128 SMs busy, so its
// reduction dimension is split over a thread-block cluster of `split` CTAs
// (one per SM, split <= 8, the largest for which every cluster is resident at
// once): each CTA streams
// its K range of the block through a TMA ring into tcgen05.mma.kind::f16
// with the fp32 partial in TMEM, writes the partial to its shared memory,
// and after a cluster barrier every CTA sums its share of the block's rows
// over all partials through distributed shared memory, adds the residual and
// rounds once.  No global workspace, no atomics.
//
//   warp 0      TMA: W tile 128 x 64 and X tile NT x 64 (128-byte swizzle)
//               per stage of a 6-stage ring
//   warp 1      TMEM (NT columns, at least 32); one lane issues the MMAs
//   warps 2-5   TMEM -> shared memory (thread = W row)
//   all warps   cluster reduction, residual add, bf16 stores
#include "kernels.h"
#include "tc.cuh"

namespace gqa {
namespace {

#ifndef GQA_OPROJ_MAX_SPLIT
#define GQA_OPROJ_MAX_SPLIT 8
#endif
constexpr int BM = 128, BK = 64, STAGES = 6, THREADS = 192, kMaxSplit = GQA_OPROJ_MAX_SPLIT;

template <int NT>
struct SmallCfg {
  static constexpr int A_BYTES = BM * BK * 2;          // W tile, 16 KB
  static constexpr int B_BYTES = NT * BK * 2;          // X tile
  static constexpr int STAGE = A_BYTES + B_BYTES;      // a multiple of 1024
  static constexpr int RED_OFF = STAGES * STAGE;       // fp32 partial [NT][BM]
  static constexpr int BAR_OFF = RED_OFF + NT * BM * 4;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static constexpr uint32_t TMEM_COLS = NT < 32 ? 32 : NT;
  static constexpr uint32_t IDESC = tc::idesc_bf16(BM, NT, false, false);
  static_assert(STAGE % 1024 == 0, "stage tiles stay 1024-byte aligned");
};

struct SmallBars {
  uint64_t full[STAGES], empty[STAGES], acc_full, drain;
  uint32_t tmem_base;
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

template <int NT>
__global__ void __launch_bounds__(THREADS, 1)
oproj_smallt_kernel(const __grid_constant__ CUtensorMap tmw, const __grid_constant__ CUtensorMap tmx, OprojParams p,
                    int split, int n_kb) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  using C = SmallCfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SmallBars* bars = reinterpret_cast<SmallBars*>(smem + C::BAR_OFF);
  float* red = reinterpret_cast<float*>(smem + C::RED_OFF);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int* err = p.err;

  const int rank = (int)cluster_ctarank();
  const int m0 = (blockIdx.x / split) * BM;
  const int kb_lo = rank * n_kb / split, kb_hi = (rank + 1) * n_kb / split;   // split <= n_kb: never empty
  const int nk = kb_hi - kb_lo;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmw);
    tc::prefetch_tmap(&tmx);
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  bool ok = true;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int i = 0;
      for (; i < nk; ++i) {
        const int st = i % STAGES;
        if (!mbar_wait(&bars->empty[st], ((i / STAGES) & 1) ^ 1, err)) break;
        uint8_t* sa = smem + st * C::STAGE;
        mbar_arrive_expect_tx(&bars->full[st], C::STAGE);
        tc::tma_load_2d(sa, &tmw, (kb_lo + i) * BK, m0, &bars->full[st]);
        tc::tma_load_2d(sa + C::A_BYTES, &tmx, (kb_lo + i) * BK, 0, &bars->full[st]);
      }
      // every issued copy has landed before the CTA may exit
      for (int k = i - 1; k >= 0 && k >= i - STAGES; --k) mbar_wait_drain(&bars->full[k % STAGES], (k / STAGES) & 1, err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int i = 0; i < nk; ++i) {
        const int st = i % STAGES;
        if (!mbar_wait(&bars->full[st], (i / STAGES) & 1, err)) break;
        tc::fence_after_sync();
        const uint32_t sa = smem_u32(smem + st * C::STAGE), sb = sa + C::A_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          tc::mma_bf16_ss(tmem, tc::sdesc_sw128(sa + k * 32, 16, 1024), tc::sdesc_sw128(sb + k * 32, 16, 1024), C::IDESC,
                          (i | k) != 0);
        tc::mma_commit(&bars->empty[st]);
      }
      tc::mma_commit(&bars->acc_full);
      tc::mma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, err);
    }
  } else {
    // ------------------------------------------------------------ TMEM -> shared memory
    const int row = (warp & 3) * 32 + lane;
    ok = __all_sync(0xffffffffu, mbar_wait(&bars->acc_full, 0, err));
    tc::fence_after_sync();
#pragma unroll
    for (int c = 0; c < NT / 16; ++c) {
      uint32_t v[16];
      if (ok) {
        tc::tmem_ld16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + c * 16, v);
        tc::tmem_ld_wait();
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = 0u;
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) red[(c * 16 + k) * BM + row] = __uint_as_float(v[k]);
    }
  }

  // every CTA's partial is in its shared memory; sum this CTA's share of rows
  tc::fence_before_sync();
  __syncwarp();   // the single-lane roles rejoin their warps before the aligned barrier
  tc::cluster_sync();
  const int rows = ((BM + split - 1) / split + 3) / 4 * 4;   // a multiple of 4 rows per CTA
  const int r0 = rank * rows, r1 = min(BM, r0 + rows);
  const int T = p.T;
  const __nv_bfloat16* res = static_cast<const __nv_bfloat16*>(p.residual);
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  if (r1 > r0) {
    const int quads = (r1 - r0) / 4;
    const uint32_t red_u = smem_u32(red);
    for (int e = threadIdx.x; e < quads * T; e += THREADS) {
      const int tok = e / quads, r = r0 + 4 * (e % quads);
      const int n = m0 + r;
      if (n >= p.N) continue;   // N % 8 == 0: a quad is wholly inside or outside
      // every CTA's partial: all remote loads issued before the first add
      float4 part[kMaxSplit];
      const uint32_t a = red_u + (uint32_t)(tok * BM + r) * 4u;
#pragma unroll
      for (int q = 0; q < kMaxSplit; ++q)
        if (q < split) part[q] = tc::ld_dsmem_f32x4(tc::mapa_shared(a, (uint32_t)q));
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < kMaxSplit; ++q)
        if (q < split) {
          acc.x += part[q].x;
          acc.y += part[q].y;
          acc.z += part[q].z;
          acc.w += part[q].w;
        }
      const size_t o = (size_t)tok * p.N + n;
      if (res) {
        const uint2 rv = *reinterpret_cast<const uint2*>(res + o);
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&rv.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&rv.y);
        acc.x += __low2float(a);
        acc.y += __high2float(a);
        acc.z += __low2float(b);
        acc.w += __high2float(b);
      }
      uint2 w;
      w.x = pack_bf16x2(acc.x, acc.y);
      w.y = pack_bf16x2(acc.z, acc.w);
      *reinterpret_cast<uint2*>(out + o) = w;
    }
  }
  // no CTA leaves while another may still read its shared memory
  tc::cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int NT>
cudaError_t launch_nt(const OprojParams& p, int num_sms, cudaStream_t st) {
  using C = SmallCfg<NT>;
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = smem_attr_once(attr_set, reinterpret_cast<const void*>(oproj_smallt_kernel<NT>), C::SMEM);
      e != cudaSuccess)
    return e;
  const int n_mblk = (p.N + BM - 1) / BM;
  const int n_kb = (p.K + BK - 1) / BK;
  // The largest split whose clusters all fit on the GPU at once (measured on
  // B200: at most 15 clusters of 8 are resident, so 16 row blocks x 8 would
  // take two waves), found once per device and split from the occupancy API.
  static std::atomic<int> max_clusters[64][kMaxSplit + 1];   // 0 unknown, else clusters + 1
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    dev = -1;
  }
  int split = 1;
  for (int sp = kMaxSplit; sp >= 1; --sp) {
    if (sp > n_kb || n_mblk * sp > num_sms) continue;
    int fit = dev >= 0 ? max_clusters[dev][sp].load(std::memory_order_relaxed) - 1 : -1;
    if (fit < 0) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3((unsigned)(n_mblk * sp), 1, 1);
      q.blockDim = dim3(THREADS, 1, 1);
      q.dynamicSmemBytes = C::SMEM;
      cudaLaunchAttribute qa[1];
      qa[0].id = cudaLaunchAttributeClusterDimension;
      qa[0].val.clusterDim.x = (unsigned)sp;
      qa[0].val.clusterDim.y = 1;
      qa[0].val.clusterDim.z = 1;
      q.attrs = qa;
      q.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&fit, oproj_smallt_kernel<NT>, &q) != cudaSuccess) {
        cudaGetLastError();
        fit = 0;
      }
      if (dev >= 0) max_clusters[dev][sp].store(fit + 1, std::memory_order_relaxed);
    }
    if (fit >= n_mblk) {
      split = sp;
      break;
    }
  }
  CUtensorMap tw, tx;
  if (!make_tmap_bf16_2d(&tw, p.w, p.K, p.N, (uint64_t)p.K * 2, BK, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tx, p.x, p.K, p.T, (uint64_t)p.K * 2, BK, NT)) return cudaErrorInvalidValue;
  return launch_ex(oproj_smallt_kernel<NT>, dim3((unsigned)(n_mblk * split)), dim3(THREADS), C::SMEM, st,
                   (unsigned)split, tw, tx, p, split, n_kb);
}

}  // namespace

cudaError_t launch_oproj_smallt(const OprojParams& p, int num_sms, cudaStream_t st) {
  if (p.T <= 16) return launch_nt<16>(p, num_sms, st);
  if (p.T <= 32) return launch_nt<32>(p, num_sms, st);
  if (p.T <= 64) return launch_nt<64>(p, num_sms, st);
  return cudaErrorInvalidValue;
}

}  // namespace gqa
