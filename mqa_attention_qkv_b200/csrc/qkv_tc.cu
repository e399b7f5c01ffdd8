// The layer's two projection GEMMs on the Blackwell tensor cores (bf16):
//   * the fused QKV projection, with RoPE and the head-major scatter in the
//     epilogue (steps a1-a3): Y[T, N] = X[T, D] . W[N, D]^T with
//     N = (nh + 2 nkv) * hd, the fused W_qkv of "Optimize LlamaAttention by
//     fusing QKV projections" (huggingface/transformers #40092);
//   * the output projection with the residual add in the epilogue:
//     out[T, hidden] = attn[T, nh*hd] . W_o^T + residual (the custom-op
//     overhead gist's LlamaAttention.forward ends in its output projection,
//     and its decoder layer adds the residual stream).
// Both operands are K-major (the reduction dimension contiguous), which is
// what tcgen05 reads natively.  One kernel template serves both; only the
// epilogue differs.
//
// Persistent kernel, one CTA per SM, 6 warps:
//   warp 0      TMA producer: X and W tiles (128 x 64 and 256 x 64, 128-byte
//               swizzle) into a 4-stage shared-memory ring
//   warp 1      allocates 512 TMEM columns; one lane issues the
//               tcgen05.mma.kind::f16 (M=128, N=256, K=16) into one of two
//               fp32 accumulators in TMEM (double buffered across tiles)
//   warps 2-5   epilogue: thread = token row; tcgen05.ld the accumulator.
//               QKV: rotate q/k feature pairs (i, i + hd/2) in fp32, round to
//               bf16 once and store each head straight to q_out
//               [B, nh, S, hd] or to the cache row [b, j, position]; tiles are
//               128 tokens x 256 fused features, i.e. whole heads, so a
//               rotation pair never leaves the thread that holds it.
//               Output projection: add the residual row in fp32, round once.
#include "kernels.h"
#include "tc.cuh"

namespace gqa {
namespace {

constexpr int BM = 128, BK = 64, MAX_STAGES = 8;
constexpr int THREADS = 192;

// Tile width and ring depth.  Wide (N 256, 4 stages) for many-token
// problems; narrow (N 64 or 128, 8 or 6 stages) when the wide tiles would
// leave most SMs idle (a 128-token projection is 10 tiles wide): more, thinner
// tiles and more bytes in flight per SM.
template <int BN_, int STAGES_>
struct GemmCfg {
  static constexpr int BN = BN_, STAGES = STAGES_;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;     // two accumulators
  static constexpr uint32_t IDESC = tc::idesc_bf16(BM, BN, false, false);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 1024 /*barriers, tables*/;
  static_assert(STAGES <= MAX_STAGES, "barrier arrays");
};

template <class P>
struct TcArgs {
  P p;
  int T, n_heads_total, num_n, num_tiles, num_kb;
};

struct Bars {
  uint64_t full[MAX_STAGES], empty[MAX_STAGES], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int abort;
  double inv_freq[64];
};

// Epilogue of the QKV projection: RoPE on q/k, head-major scatter.  One
// thread owns token row `row` of the 128 x 256 tile at (m0, n0); `tbase` is
// its TMEM lane in the accumulator buffer.
template <int HD>
struct QkvEpilogue {
  using Params = QkvParams;
  __device__ static void init(const Params& p, Bars* bars) {
    if (threadIdx.x >= 64 && threadIdx.x < 64 + HD / 2)
      bars->inv_freq[threadIdx.x - 64] = rope_inv_freq(threadIdx.x - 64, HD, p.theta);
  }
  template <int BN>
  __device__ static void tile(const TcArgs<Params>& a, const Bars* bars, uint32_t tbase, int m0, int n0, int row) {
    constexpr int HALF = HD / 2, CHUNKS = HALF / 16, HEADS = BN / HD;
    static_assert(BN % HD == 0, "tiles hold whole heads");
    const Params& p = a.p;
    int* err = p.err;
    const int t = m0 + row;
    const bool valid = t < a.T;
    int b = 0, s = 0, pos = 0;
    if (valid) {
      b = t / p.S;
      s = t - b * p.S;
      pos = p.pos[t];
    }
    const bool pos_ok = pos >= 0 && pos < p.cap;
    const int hb0 = n0 / HD;
#pragma unroll 1
    for (int c = 0; c < CHUNKS; ++c) {
      float cs[16], sn[16];
      if (valid) {
#pragma unroll
        for (int k = 0; k < 16; ++k) rope_cos_sin(pos, bars->inv_freq[c * 16 + k], &cs[k], &sn[k]);
      }
#pragma unroll 1
      for (int hh = 0; hh < HEADS; ++hh) {
        const int hb = hb0 + hh;
        if (hb >= a.n_heads_total) break;  // ragged N tail: uniform over the CTA
        uint32_t lo[16], hi[16];
        __syncwarp();  // the .sync.aligned TMEM load needs the whole warp converged
        tc::tmem_ld16(tbase + hh * HD + c * 16, lo);
        tc::tmem_ld16(tbase + hh * HD + HALF + c * 16, hi);
        tc::tmem_ld_wait();
        if (!valid) continue;
        const bool is_q = hb < p.nh, is_k = !is_q && hb < p.nh + p.nkv;
        __nv_bfloat16* dst;
        if (is_q) {
          dst = static_cast<__nv_bfloat16*>(p.q_out) + (((size_t)b * p.nh + hb) * p.S + s) * HD;
        } else {
          if (!pos_ok) {
            if (c == 0) raise_error(err, GQA_DEVERR_POSITION_RANGE);
            continue;
          }
          const int j = is_k ? hb - p.nh : hb - p.nh - p.nkv;
          dst = static_cast<__nv_bfloat16*>(is_k ? p.k_cache : p.v_cache) +
                (((size_t)b * p.nkv + j) * p.cap + pos) * HD;
        }
        uint32_t olo[8], ohi[8];
        if (is_q || is_k) {
#pragma unroll
          for (int k = 0; k < 16; k += 2) {
            const float x0 = __uint_as_float(lo[k]), y0 = __uint_as_float(hi[k]);
            const float x1 = __uint_as_float(lo[k + 1]), y1 = __uint_as_float(hi[k + 1]);
            olo[k / 2] = pack_bf16x2(x0 * cs[k] - y0 * sn[k], x1 * cs[k + 1] - y1 * sn[k + 1]);
            ohi[k / 2] = pack_bf16x2(y0 * cs[k] + x0 * sn[k], y1 * cs[k + 1] + x1 * sn[k + 1]);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; k += 2) {
            olo[k / 2] = pack_bf16x2(__uint_as_float(lo[k]), __uint_as_float(lo[k + 1]));
            ohi[k / 2] = pack_bf16x2(__uint_as_float(hi[k]), __uint_as_float(hi[k + 1]));
          }
        }
        tc::st_global_v4(dst + c * 16, olo[0], olo[1], olo[2], olo[3]);
        tc::st_global_v4(dst + c * 16 + 8, olo[4], olo[5], olo[6], olo[7]);
        tc::st_global_v4(dst + HALF + c * 16, ohi[0], ohi[1], ohi[2], ohi[3]);
        tc::st_global_v4(dst + HALF + c * 16 + 8, ohi[4], ohi[5], ohi[6], ohi[7]);
      }
    }
  }
};

// Epilogue of the output projection: out = acc + residual, rounded once.
// Columns are stored in 8-wide vectors; a vector past N (N % 8 == 0) is
// skipped, so a ragged N tail needs no masking inside a vector.
struct ResidualEpilogue {
  using Params = OprojParams;
  __device__ static void init(const Params&, Bars*) {}
  template <int BN>
  __device__ static void tile(const TcArgs<Params>& a, const Bars*, uint32_t tbase, int m0, int n0, int row) {
    const Params& p = a.p;
    const int t = m0 + row;
    const bool valid = t < a.T;
    const __nv_bfloat16* res = static_cast<const __nv_bfloat16*>(p.residual);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + (size_t)t * p.N;
#pragma unroll 1
    for (int c = 0; c < BN / 16; ++c) {
      const int n = n0 + c * 16;
      if (n >= p.N) break;   // uniform over the CTA
      uint32_t v[16];
      __syncwarp();
      tc::tmem_ld16(tbase + c * 16, v);
      tc::tmem_ld_wait();
      if (!valid) continue;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (n + 8 * h >= p.N) break;
        float f[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(v[8 * h + k]);
        if (res) {
          const uint4 r = *reinterpret_cast<const uint4*>(res + (size_t)t * p.N + n + 8 * h);
          const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&rw[k]);
            f[2 * k] += __low2float(b2);
            f[2 * k + 1] += __high2float(b2);
          }
        }
        tc::st_global_v4(out + n + 8 * h, pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                         pack_bf16x2(f[6], f[7]));
      }
    }
  }
};

template <class Epi, class Cfg>
__global__ void __launch_bounds__(THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
               TcArgs<typename Epi::Params> a) {
  constexpr int BN = Cfg::BN, STAGES = Cfg::STAGES, A_BYTES = Cfg::A_BYTES, STAGE_BYTES = Cfg::STAGE_BYTES;
  constexpr int TMEM_COLS = Cfg::TMEM_COLS;
  constexpr uint32_t IDESC = Cfg::IDESC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int* err = a.p.err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], 4);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  Epi::init(a.p, bars);
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmx);
    tc::prefetch_tmap(&tmw);
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, TMEM_COLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x) {
        const int m0 = (tile / a.num_n) * BM, n0 = (tile % a.num_n) * BN;
        for (int kb = 0; kb < a.num_kb; ++kb) {
          if (!mbar_wait(&bars->empty[stage], phase ^ 1, err)) { ok = false; break; }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&bars->full[stage], STAGE_BYTES);
          tc::tma_load_2d(sa, &tmx, kb * BK, m0, &bars->full[stage]);
          tc::tma_load_2d(sa + A_BYTES, &tmw, kb * BK, n0, &bars->full[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) atomicExch(&bars->abort, 1);
      // every issued load has landed before the CTA may exit
      for (int s = 0; s < STAGES; ++s) {
        int st = (stage + s) % STAGES;
        uint32_t ph = (st < stage) ? phase : phase ^ 1;  // phase of the last load issued into st
        mbar_wait_drain(&bars->full[st], ph, err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; ok && tile < a.num_tiles; tile += gridDim.x, ++it) {
        const int buf = it & 1;
        if (!mbar_wait(&bars->acc_empty[buf], ((it >> 1) & 1) ^ 1, err)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t d = tmem + buf * BN;
        for (int kb = 0; kb < a.num_kb; ++kb) {
          if (!mbar_wait(&bars->full[stage], phase, err)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            tc::mma_bf16_ss(d, tc::sdesc_sw128(sa + k * 32, 16, 1024), tc::sdesc_sw128(sb + k * 32, 16, 1024),
                            IDESC, (kb | k) != 0);
          }
          tc::mma_commit(&bars->empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc::mma_commit(&bars->acc_full[buf]);
      }
      if (!ok) atomicExch(&bars->abort, 1);
      // all MMAs done before TMEM is released
      tc::mma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, err);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x, ++it) {
      const int buf = it & 1;
      const bool got = mbar_wait(&bars->acc_full[buf], (it >> 1) & 1, err);
      if (!__all_sync(0xffffffffu, got)) break;
      tc::fence_after_sync();
      const int m0 = (tile / a.num_n) * BM, n0 = (tile % a.num_n) * BN;
      const uint32_t tbase = tmem + ((uint32_t)(q4 * 32) << 16) + buf * BN;
      Epi::template tile<BN>(a, bars, tbase, m0, n0, row);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <class Epi, class Cfg>
cudaError_t launch_cfg(const typename Epi::Params& p, const void* x, const void* w, int T, int K, int N,
                       int n_heads_total, int num_sms, cudaStream_t st) {
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = smem_attr_once(attr_set, reinterpret_cast<const void*>(gemm_tc_kernel<Epi, Cfg>),
                                     Cfg::SMEM_BYTES);
      e != cudaSuccess)
    return e;
  TcArgs<typename Epi::Params> a;
  a.p = p;
  a.T = T;
  a.n_heads_total = n_heads_total;
  a.num_n = (N + Cfg::BN - 1) / Cfg::BN;
  a.num_tiles = ((T + BM - 1) / BM) * a.num_n;
  a.num_kb = (K + BK - 1) / BK;
  CUtensorMap tx, tw;
  if (!make_tmap_bf16_2d(&tx, x, K, T, (uint64_t)K * 2, BK, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tw, w, K, N, (uint64_t)K * 2, BK, Cfg::BN)) return cudaErrorInvalidValue;
  const int grid = a.num_tiles < num_sms ? a.num_tiles : num_sms;
  gemm_tc_kernel<Epi, Cfg><<<grid, THREADS, Cfg::SMEM_BYTES, st>>>(tx, tw, a);
  return cudaGetLastError();
}

// Wide tiles unless they would leave more than half of the SMs idle; then
// the narrowest tile that still holds whole heads (`min_bn`).
template <class Epi, int MIN_BN>
cudaError_t launch_gemm(const typename Epi::Params& p, const void* x, const void* w, int T, int K, int N,
                        int n_heads_total, int num_sms, cudaStream_t st) {
  const long long wide_tiles = (long long)((T + BM - 1) / BM) * ((N + 255) / 256);
  if (2 * wide_tiles >= num_sms) return launch_cfg<Epi, GemmCfg<256, 4>>(p, x, w, T, K, N, n_heads_total, num_sms, st);
  if constexpr (MIN_BN <= 64)
    return launch_cfg<Epi, GemmCfg<64, 8>>(p, x, w, T, K, N, n_heads_total, num_sms, st);
  else
    return launch_cfg<Epi, GemmCfg<128, 6>>(p, x, w, T, K, N, n_heads_total, num_sms, st);
}

}  // namespace

cudaError_t launch_qkv_tc(const QkvParams& p, int num_sms, cudaStream_t st) {
  const int T = p.B * p.S, heads = p.nh + 2 * p.nkv, N = heads * p.hd;
  switch (p.hd) {
    case 32: return launch_gemm<QkvEpilogue<32>, 64>(p, p.x, p.w, T, p.hidden, N, heads, num_sms, st);
    case 64: return launch_gemm<QkvEpilogue<64>, 64>(p, p.x, p.w, T, p.hidden, N, heads, num_sms, st);
    case 128: return launch_gemm<QkvEpilogue<128>, 128>(p, p.x, p.w, T, p.hidden, N, heads, num_sms, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_oproj_tc(const OprojParams& p, int num_sms, cudaStream_t st) {
  return launch_gemm<ResidualEpilogue, 64>(p, p.x, p.w, p.T, p.K, p.N, 0, num_sms, st);
}

}  // namespace gqa
