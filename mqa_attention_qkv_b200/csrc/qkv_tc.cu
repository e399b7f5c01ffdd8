// Fused QKV projection on the Blackwell tensor cores, with RoPE and the
// head-major scatter in the epilogue (steps a1-a3, bf16).
//
// Y[T, N] = X[T, D] . W[N, D]^T, N = (nh + 2 nkv) * hd, from the fused
// W_qkv of "Optimize LlamaAttention by fusing QKV projections"
// (huggingface/transformers #40092).  Both operands are K-major (D
// contiguous), which is what tcgen05 reads natively.
//
// Persistent kernel, one CTA per SM, 6 warps:
//   warp 0      TMA producer: X and W tiles (128 x 64 and 256 x 64, 128-byte
//               swizzle) into a 4-stage shared-memory ring
//   warp 1      allocates 512 TMEM columns; one lane issues the
//               tcgen05.mma.kind::f16 (M=128, N=256, K=16) into one of two
//               fp32 accumulators in TMEM (double buffered across tiles)
//   warps 2-5   epilogue: thread = token row; tcgen05.ld the accumulator,
//               rotate q/k feature pairs (i, i + hd/2) in fp32, round to
//               bf16 once and store each head straight to q_out
//               [B, nh, S, hd] or to the cache row [b, j, position]
// Tiles are 128 tokens x 256 fused features, i.e. whole heads, so a
// rotation pair never leaves the thread that holds it.
#include "kernels.h"
#include "tc.cuh"

namespace gqa {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * BN;
constexpr int THREADS = 192;
constexpr uint32_t IDESC = tc::idesc_bf16(BM, BN, false, false);
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 1024 /*barriers, tables*/;

struct TcArgs {
  QkvParams p;
  int T, n_heads_total, num_n, num_tiles, num_kb;
};

struct Bars {
  uint64_t full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int abort;
  double inv_freq[64];
};

template <int HD>
__global__ void __launch_bounds__(THREADS, 1)
qkv_tc_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw, TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const QkvParams& p = a.p;
  int* err = p.err;

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
  if (threadIdx.x >= 64 && threadIdx.x < 64 + HD / 2)
    bars->inv_freq[threadIdx.x - 64] = rope_inv_freq(threadIdx.x - 64, HD, p.theta);
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
        mbar_wait(&bars->full[st], ph, err);
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
      mbar_wait(&bars->drain, 0, err);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int HALF = HD / 2, CHUNKS = HALF / 16, HEADS = BN / HD;
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x, ++it) {
      const int buf = it & 1;
      const bool got = mbar_wait(&bars->acc_full[buf], (it >> 1) & 1, err);
      if (!__all_sync(0xffffffffu, got)) break;
      tc::fence_after_sync();
      const int m0 = (tile / a.num_n) * BM, n0 = (tile % a.num_n) * BN;
      const int t = m0 + row;
      const bool valid = t < a.T;
      int b = 0, s = 0, pos = 0;
      if (valid) {
        b = t / p.S;
        s = t - b * p.S;
        pos = p.pos[t];
      }
      const bool pos_ok = pos >= 0 && pos < p.cap;
      const uint32_t tbase = tmem + ((uint32_t)(q4 * 32) << 16) + buf * BN;
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

template <int HD>
cudaError_t launch_hd(const CUtensorMap& tx, const CUtensorMap& tw, const TcArgs& a, int grid, cudaStream_t st) {
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = smem_attr_once(attr_set, reinterpret_cast<const void*>(qkv_tc_kernel<HD>), SMEM_BYTES);
      e != cudaSuccess)
    return e;
  qkv_tc_kernel<HD><<<grid, THREADS, SMEM_BYTES, st>>>(tx, tw, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qkv_tc(const QkvParams& p, int num_sms, cudaStream_t st) {
  TcArgs a;
  a.p = p;
  a.T = p.B * p.S;
  a.n_heads_total = p.nh + 2 * p.nkv;
  const int N = a.n_heads_total * p.hd;
  a.num_n = (N + BN - 1) / BN;
  a.num_tiles = ((a.T + BM - 1) / BM) * a.num_n;
  a.num_kb = (p.hidden + BK - 1) / BK;
  CUtensorMap tx, tw;
  if (!make_tmap_bf16_2d(&tx, p.x, p.hidden, a.T, (uint64_t)p.hidden * 2, BK, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tw, p.w, p.hidden, N, (uint64_t)p.hidden * 2, BK, BN)) return cudaErrorInvalidValue;
  const int grid = a.num_tiles < num_sms ? a.num_tiles : num_sms;
  switch (p.hd) {
    case 32: return launch_hd<32>(tx, tw, a, grid, st);
    case 64: return launch_hd<64>(tx, tw, a, grid, st);
    case 128: return launch_hd<128>(tx, tw, a, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gqa
