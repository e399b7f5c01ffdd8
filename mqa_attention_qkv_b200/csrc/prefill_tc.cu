// Prefill attention on the Blackwell tensor cores (step a4, bf16, head_dim 64
// or 128): exact online-softmax attention in the tiled form the
// FlashAttention-3 summary recaps ("FlashAttention方式のおさらい": tiles,
// softmax rescaling, no score matrix in HBM), with grouped-query heads (MHA ->
// GQA blog, section 3.2): query head h reads KV head h / g.
//
// One CTA per (sequence b, query head h, tile of 128 query rows); causal
// tiles are scheduled longest first.  6 warps:
//   warp 0     TMA: the Q tile once, then K and V tiles of 128 keys into
//              separate rings (K is released as soon as S = QK^T is done, so
//              the next K streams in while softmax still runs).  It also zeroes
//              the V rows at or beyond kv_len in the last tile, so NaN padding
//              never meets a zero probability (0 * NaN = NaN).
//   warp 1     allocates TMEM; one lane issues tcgen05.mma kind::f16:
//              S_j = Q K_j^T (M128 N128, two S buffers in TMEM) one tile ahead
//              of O += P_j V_j (M128 N=hd, V read MN-major from its TMA tile).
//   warps 2-5  softmax, thread = query row: tcgen05.ld the S row, mask, row
//              max, P = 2^(s - m) (ex2.approx), row sum in fp32, P rounded to
//              bf16 into a 128-byte-swizzled shared tile for the next MMA.
//              O stays in TMEM.  It is rescaled (tcgen05.ld/st) only when a
//              row's max grows by more than 8 in log2 units; otherwise the
//              stale max is kept, which is exact after the final 1/l and keeps
//              P <= 2^8.  At the end O / l is rounded once to bf16 and stored
//              to out[b, s, h, :].
#include "kernels.h"
#include "tc.cuh"

namespace gqa {
namespace {

constexpr int BQ = 128, BKV = 128, THREADS = 192;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int HD>
struct Cfg {
  static constexpr int KS = HD == 128 ? 2 : 3;   // K ring depth
  static constexpr int VS = HD == 128 ? 2 : 3;   // V ring depth
  static constexpr int TILE_BYTES = 128 * HD * 2;           // Q, K or V tile
  static constexpr int P_BYTES = BQ * BKV * 2;              // one P buffer
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE_BYTES;
  static constexpr int V_OFF = K_OFF + KS * TILE_BYTES;
  static constexpr int P_OFF = V_OFF + VS * TILE_BYTES;
  static constexpr int BAR_OFF = P_OFF + 2 * P_BYTES;
  static constexpr int SMEM = BAR_OFF + 1024 + 1024;        // barriers + alignment slack
  static constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, false, false);
  static constexpr uint32_t IDESC_O = tc::idesc_bf16(128, HD, false, true);
};

struct Bars {
  uint64_t q_full, v_clean, drain;
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t s_full[2], s_empty[2], p_full[2], o_done[2];
  uint32_t tmem_base;
  int max_pos;
};

struct TcPrefillArgs {
  PrefillParams p;
  int n_qt;  // query tiles per (b, h)
};

// TMEM columns: S buffers at 0 and 128, O at 256.
constexpr uint32_t kTmemCols = 512, kOCol = 256;

template <int HD>
__global__ void __launch_bounds__(THREADS, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, TcPrefillArgs a) {
  using C = Cfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::BAR_OFF);
  const PrefillParams& p = a.p;
  int* err = p.err;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---- work unit: longest causal tiles first, heads of a KV group adjacent
  const int bh_count = p.B * p.nh;
  const int u = blockIdx.x;
  const int qt = a.n_qt - 1 - u / bh_count;
  const int b = (u % bh_count) / p.nh;
  const int h = u % p.nh;
  const int g = p.nh / p.nkv;
  const int j = h / g;
  const int s0 = qt * BQ;

  int kv_len = p.kv_lens[b];
  if (kv_len > p.cap || kv_len < 0) {
    if (threadIdx.x == 0) raise_error(err, GQA_DEVERR_KVLEN_RANGE);
    kv_len = kv_len > p.cap ? p.cap : 0;
  }

  // ---- prologue
  const int row = (warp & 3) * 32 + lane;  // softmax/epilogue row (warps 2-5)
  int my_pos = 0, my_lim = 0;
  bool my_valid = false;
  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->v_clean, 1);
    mbar_init(&bars->drain, 1);
    for (int i = 0; i < 3; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_empty[i], 4);
      mbar_init(&bars->p_full[i], 4);
      mbar_init(&bars->o_done[i], 1);
    }
    bars->max_pos = -1;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, kTmemCols);
  __syncthreads();
  if (warp >= 2) {
    const int s = s0 + row;
    my_valid = s < p.S;
    if (my_valid) {
      my_pos = p.q_pos ? p.q_pos[(size_t)b * p.S + s] : kv_len - p.S + s;
      my_lim = p.causal ? max(0, min(kv_len, my_pos + 1)) : kv_len;
      atomicMax(&bars->max_pos, my_lim);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  const int kv_hi = bars->max_pos < 0 ? 0 : bars->max_pos;   // keys [0, kv_hi) are visible to some row
  const int n_kv = (kv_hi + BKV - 1) / BKV;
  const bool sanitize = n_kv > 0 && kv_len < n_kv * BKV;     // last tile holds rows >= kv_len
  const int kv_row0 = (b * p.nkv + j) * p.cap;

  uint8_t* sQ = smem + C::Q_OFF;
  uint8_t* sK = smem + C::K_OFF;
  uint8_t* sV = smem + C::V_OFF;
  uint8_t* sP = smem + C::P_OFF;

  if (warp == 0) {
    // ================================================================ TMA
    bool ok = true;
    if (lane == 0 && n_kv > 0) {
      mbar_arrive_expect_tx(&bars->q_full, C::TILE_BYTES);
      const int qrow = (b * p.nh + h) * p.S + s0;
      for (int c = 0; c < HD / 64; ++c) tc::tma_load_2d(sQ + c * 16384, &tmq, c * 64, qrow, &bars->q_full);
      auto load_k = [&](int t) {
        const int st = t % C::KS;
        if (!mbar_wait(&bars->k_empty[st], ((t / C::KS) & 1) ^ 1, err)) return false;
        mbar_arrive_expect_tx(&bars->k_full[st], C::TILE_BYTES);
        for (int c = 0; c < HD / 64; ++c)
          tc::tma_load_2d(sK + st * C::TILE_BYTES + c * 16384, &tmk, c * 64, kv_row0 + t * BKV, &bars->k_full[st]);
        return true;
      };
      auto load_v = [&](int t) {
        const int st = t % C::VS;
        if (!mbar_wait(&bars->v_empty[st], ((t / C::VS) & 1) ^ 1, err)) return false;
        mbar_arrive_expect_tx(&bars->v_full[st], C::TILE_BYTES);
        for (int c = 0; c < HD / 64; ++c)
          tc::tma_load_2d(sV + st * C::TILE_BYTES + c * 16384, &tmv, c * 64, kv_row0 + t * BKV, &bars->v_full[st]);
        return true;
      };
      ok = load_k(0);
      for (int t = 0; ok && t < n_kv; ++t) {
        if (t + 1 < n_kv) ok = load_k(t + 1);
        if (ok) ok = load_v(t);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok && sanitize) {
      // zero V rows >= kv_len of the last tile (whole 128-byte rows: the
      // swizzle only permutes 16-byte chunks inside a row)
      const int t = n_kv - 1, st = t % C::VS;
      const bool landed = mbar_wait(&bars->v_full[st], (t / C::VS) & 1, err);
      if (__all_sync(0xffffffffu, landed)) {
        const int r0 = max(0, kv_len - t * BKV);
        uint8_t* vt = sV + st * C::TILE_BYTES;
        for (int c = 0; c < HD / 64; ++c)
          for (int r = r0 + lane / 8; r < BKV; r += 4)
            *reinterpret_cast<uint4*>(vt + c * 16384 + r * 128 + (lane % 8) * 16) = make_uint4(0, 0, 0, 0);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->v_clean);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    if (lane == 0 && n_kv > 0) {
      bool ok = mbar_wait(&bars->q_full, 0, err);
      const uint32_t q_addr = smem_u32(sQ);
      auto issue_s = [&](int t) {
        const int st = t % C::KS;
        if (!mbar_wait(&bars->k_full[st], (t / C::KS) & 1, err)) return false;
        if (t >= 2 && !mbar_wait(&bars->s_empty[t & 1], ((t >> 1) & 1) ^ 1, err)) return false;
        tc::fence_after_sync();
        const uint32_t k_addr = smem_u32(sK + st * C::TILE_BYTES);
        const uint32_t d = tmem + (t & 1) * 128;
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (k / 4) * 16384 + (k % 4) * 32;
          tc::mma_bf16_ss(d, tc::sdesc_sw128(q_addr + off, 16, 1024), tc::sdesc_sw128(k_addr + off, 16, 1024),
                          C::IDESC_S, k != 0);
        }
        tc::mma_commit(&bars->k_empty[st]);
        tc::mma_commit(&bars->s_full[t & 1]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int t = 0; ok && t < n_kv; ++t) {
        if (t + 1 < n_kv && !(ok = issue_s(t + 1))) break;
        const int vs = t % C::VS;
        if (!mbar_wait(&bars->p_full[t & 1], (t >> 1) & 1, err)) { ok = false; break; }
        if (!mbar_wait(&bars->v_full[vs], (t / C::VS) & 1, err)) { ok = false; break; }
        if (sanitize && t == n_kv - 1 && !mbar_wait(&bars->v_clean, 0, err)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t p_addr = smem_u32(sP + (t & 1) * C::P_BYTES);
        const uint32_t v_addr = smem_u32(sV + vs * C::TILE_BYTES);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k) {
          const uint32_t a_off = (k / 4) * 16384 + (k % 4) * 32;   // P: K-major, 64-key blocks
          const uint32_t b_off = k * 16 * 128;                      // V: 16 keys x 128-byte rows
          tc::mma_bf16_ss(tmem + kOCol, tc::sdesc_sw128(p_addr + a_off, 16, 1024),
                          tc::sdesc_sw128(v_addr + b_off, 16384, 1024), C::IDESC_O, (t | k) != 0);
        }
        tc::mma_commit(&bars->v_empty[vs]);
        tc::mma_commit(&bars->o_done[t & 1]);
      }
      tc::mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, err);
    }
  } else {
    // ================================================================ softmax
    const float scale_log2 = 1.4426950408889634f * rsqrtf((float)HD);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < n_kv; ++t) {
      const int k0 = t * BKV;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[t & 1], (t >> 1) & 1, err));
      if (!ok) break;
      tc::fence_after_sync();
      float s[BKV];
#pragma unroll
      for (int c = 0; c < BKV / 16; ++c) {
        uint32_t r[16];
        tc::tmem_ld16(tmem + lane_base + (t & 1) * 128 + c * 16, r);
#pragma unroll
        for (int i = 0; i < 16; ++i) s[c * 16 + i] = __uint_as_float(r[i]);
      }
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_empty[t & 1]);

      // scale to log2 units, mask, row max
      float mx = -INFINITY;
      if (k0 + BKV <= my_lim) {
#pragma unroll
        for (int i = 0; i < BKV; ++i) {
          s[i] *= scale_log2;
          mx = fmaxf(mx, s[i]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < BKV; ++i) {
          s[i] = (k0 + i < my_lim) ? s[i] * scale_log2 : -INFINITY;
          mx = fmaxf(mx, s[i]);
        }
      }
      // lazy rescale of l and O
      float alpha = 1.f;
      if (m_used == -INFINITY) {
        m_used = mx;
      } else if (mx > m_used + kRescaleThreshold) {
        alpha = tc::ex2(m_used - mx);
        l *= alpha;
        m_used = mx;
      }
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
        // O must hold PV_{t-1} before it is scaled
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[(t - 1) & 1], ((t - 1) >> 1) & 1, err));
        if (!ok) break;
        tc::fence_after_sync();
#pragma unroll 1
        for (int c = 0; c < HD / 16; ++c) {
          uint32_t r[16];
          tc::tmem_ld16(tmem + lane_base + kOCol + c * 16, r);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tc::tmem_st16(tmem + lane_base + kOCol + c * 16, r);
        }
        tc::tmem_st_wait();
      }
      // P buffer (t & 1) is free once PV_{t-2} is done
      if (t >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[t & 1], ((t - 2) >> 1) & 1, err));
        if (!ok) break;
      }
      const float m_sub = m_used == -INFINITY ? 0.f : m_used;
      const uint32_t p_row = smem_u32(sP + (t & 1) * C::P_BYTES) + row * 128;
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < BKV / 8; ++c) {   // 16-byte chunks of 8 keys
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float p0 = tc::ex2(s[c * 8 + 2 * i] - m_sub);
          const float p1 = tc::ex2(s[c * 8 + 2 * i + 1] - m_sub);
          sum += p0 + p1;
          w[i] = pack_bf16x2(p0, p1);
        }
        const int kb = c / 8, ch = c % 8;
        tc::st_shared_v4(p_row + kb * 16384 + ((ch ^ (row & 7)) * 16), w[0], w[1], w[2], w[3]);
      }
      l += sum;
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[t & 1]);
    }

    // ---- epilogue: O / l -> out[b, s, h, :]
    if (ok && n_kv > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[(n_kv - 1) & 1], ((n_kv - 1) >> 1) & 1, err));
    tc::fence_after_sync();
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) +
                         (((size_t)b * p.S + (s0 + row)) * p.nh + h) * HD;
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
    for (int c = 0; c < HD / 16; ++c) {
      uint32_t r[16];
      if (ok && n_kv > 0) {
        __syncwarp();
        tc::tmem_ld16(tmem + lane_base + kOCol + c * 16, r);
        tc::tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = 0u;
      }
      if (my_valid) {
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          o[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
        tc::st_global_v4(dst + c * 16, o[0], o[1], o[2], o[3]);
        tc::st_global_v4(dst + c * 16 + 8, o[4], o[5], o[6], o[7]);
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int HD>
cudaError_t launch_hd(const PrefillParams& p, cudaStream_t st) {
  using C = Cfg<HD>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap tq, tk, tv;
  const uint64_t q_rows = (uint64_t)p.B * p.nh * p.S, kv_rows = (uint64_t)p.B * p.nkv * p.cap;
  if (!make_tmap_bf16_2d(&tq, p.q, HD, q_rows, HD * 2, 64, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tk, p.k_cache, HD, kv_rows, HD * 2, 64, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tv, p.v_cache, HD, kv_rows, HD * 2, 64, 128)) return cudaErrorInvalidValue;
  TcPrefillArgs a{p, (p.S + BQ - 1) / BQ};
  const long long grid = (long long)a.n_qt * p.B * p.nh;
  prefill_tc_kernel<HD><<<(unsigned)grid, THREADS, C::SMEM, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillParams& p, cudaStream_t st) {
  switch (p.hd) {
    case 64: return launch_hd<64>(p, st);
    case 128: return launch_hd<128>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gqa
