// Prefill attention for head_dim 64, two CTAs per SM (step a4, bf16).
//
// Exact tiled online softmax (FlashAttention-3 summary, recap section; GQA head
// map h -> h / g, MHA -> GQA blog section 3.2), laid out so that two CTAs
// share each SM: at head_dim 64 a KV tile costs the tensor cores half of what
// its 16K exponentials cost the MUFU unit, so the softmax of one CTA has to
// run while the other CTA's MMAs do.  Per CTA:
//   * TMEM: 256 columns = S (128 fp32 columns) | P (64) | O (64).  P, the
//     bf16 probabilities, has columns of its own and feeds the P.V MMA
//     straight from TMEM (A operand in tensor memory), so P needs no shared
//     memory and S is free as soon as the softmax warps hold it in
//     registers.
//   * shared memory: Q 16 KB + 3 K stages + 2 V stages = 96 KB.
//   * warp 0 TMA, warp 1 MMA issuer, warps 2-5 softmax (thread = query row).
// Pipeline per KV tile t: the softmax warps load S_t into registers and
// release its columns (s_free); the MMA lane then issues S_{t+1} = Q K_{t+1}^T
// at once, so the next scores are computed while the exponentials of tile t
// run, and issues P_t.V_t when P_t is stored (p_full).  The softmax stores
// P_t only after P_{t-1}.V_{t-1} has read the P columns (o_done).
// Softmax uses packed f32x2 FMA/ADD (two scores per instruction), 3-input
// max and independent accumulators so the per-row chains stay short; on
// tiles without masked keys a share of the 2^x evaluations runs as a
// polynomial on the FMA pipe (tc::exp2_poly2) next to the MUFU ex2.  O is
// rescaled in TMEM only when a row max grows by more than 2^8.
#include "kernels.h"
#include "prefill_seq.cuh"
#include "tc.cuh"

namespace gqa {
namespace {

constexpr int HD = 64, BQ = 128, BKV = 128, THREADS = 192;
constexpr int KS = 3, VS = 2;
constexpr int TILE = 128 * HD * 2;             // 16 KB
constexpr int Q_OFF = 0, K_OFF = TILE, V_OFF = K_OFF + KS * TILE, BAR_OFF = V_OFF + VS * TILE;
constexpr int SMEM = BAR_OFF + 1024 + 1024;
constexpr uint32_t kTmemCols = 256, kPCol = 128, kOCol = 192;
// Pairs out of every 8 of an unmasked row chunk whose 2^x runs on the FMA pipe.
#ifndef GQA_PAIR_POLY
#define GQA_PAIR_POLY 0
#endif
constexpr int kPoly = GQA_PAIR_POLY;
constexpr float kRescaleThreshold = 8.0f;
constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, false, false);
constexpr uint32_t IDESC_O = tc::idesc_bf16(128, HD, false, true);

struct Bars {
  uint64_t q_full, v_clean, drain, s_full, s_free, p_full, o_done;
  uint64_t k_full[KS], k_empty[KS], v_full[VS], v_empty[VS];
  uint32_t tmem_base;
  int lim_max;
};

using tc::add2;
using tc::fma2;
using tc::max3;
using tc::mma_bf16_ts;

// VARLEN: packed variable-length sequences (3-D tensor maps over
// [tokens, heads, 64 columns]); otherwise the padded layout (2-D maps over
// [rows, 64 columns]).  Both read the same 128 x 64 swizzled tiles.
template <bool VARLEN>
__global__ void __launch_bounds__(THREADS, 2)
prefill_pair_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, PrefillParams p, int n_qt) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + BAR_OFF);
  int* err = p.err;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  pdl_launch_dependents();
  pdl_wait();   // lengths, offsets and inputs may come from the kernel before this one

  const int bh_count = p.B * p.nh;
  const int u = blockIdx.x;
  const int qt = n_qt - 1 - u / bh_count;
  const int b = (u % bh_count) / p.nh;
  const int h = u % p.nh;
  const int j = h / (p.nh / p.nkv);
  const int s0 = qt * BQ;

  const SeqRange sq = prefill_seq(p, b, err);
  if (VARLEN && s0 >= sq.S) return;   // a shorter sequence: no query in this tile (whole CTA)
  const int kv_len = sq.kv_len;

  const int row = (warp & 3) * 32 + lane;
  int my_lim = 0;
  bool my_valid = false;
  // Without explicit positions a row's key limit grows with the row, so the
  // tile's key tiles follow from its last row, and thread 0 (the TMA thread)
  // can issue Q and the first two K tiles as soon as the barriers exist.
  const bool closed = p.q_pos == nullptr;
  const int rows_here = min(BQ, sq.S - s0);
  const int hi_closed = !p.causal ? kv_len : max(0, min(kv_len, kv_len - sq.S + s0 + rows_here));
  const int n_kv_closed = (hi_closed + BKV - 1) / BKV;
  const int kv_row0 = VARLEN ? 0 : (b * p.nkv + j) * p.cap;
  // failure-path testing only: the first CTA leaves one K tile unloaded
  const int skip = blockIdx.x == 0 ? p.dbg_skip_tile1 - 1 : -1;
  const int early_k = closed ? min(n_kv_closed, 2) : 0;   // K tiles issued before the role split
  uint8_t* sQ = smem + Q_OFF;
  uint8_t* sK = smem + K_OFF;
  uint8_t* sV = smem + V_OFF;
  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->v_clean, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 4);
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->o_done, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    bars->lim_max = closed ? hi_closed : -1;
    fence_mbar_init();
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
    if (closed && n_kv_closed > 0) {
      mbar_arrive_expect_tx(&bars->q_full, TILE);
      if (VARLEN)
        tc::tma_load_3d(sQ, &tmq, 0, h, sq.q0 + s0, &bars->q_full);
      else
        tc::tma_load_2d(sQ, &tmq, 0, (b * p.nh + h) * p.S + s0, &bars->q_full);
      for (int t = 0; t < early_k; ++t) {
        if (t == skip) continue;
        mbar_arrive_expect_tx(&bars->k_full[t], TILE);
        if (VARLEN)
          tc::tma_load_3d(sK + t * TILE, &tmk, 0, j, sq.k0 + t * BKV, &bars->k_full[t]);
        else
          tc::tma_load_2d(sK + t * TILE, &tmk, 0, kv_row0 + t * BKV, &bars->k_full[t]);
      }
    }
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, kTmemCols);
  __syncthreads();
  if (warp >= 2) {
    const int s = s0 + row;
    my_valid = s < sq.S;
    if (my_valid) {
      const int pos = p.q_pos ? p.q_pos[(size_t)b * p.S + s] : kv_len - sq.S + s;
      my_lim = p.causal ? max(0, min(kv_len, pos + 1)) : kv_len;
      if (!closed) atomicMax(&bars->lim_max, my_lim);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  const int kv_hi = bars->lim_max < 0 ? 0 : bars->lim_max;
  const int n_kv = (kv_hi + BKV - 1) / BKV;
  const bool sanitize = n_kv > 0 && kv_len < n_kv * BKV;

  if (warp == 0) {
    // ================================================================ TMA
    // The whole warp walks the loads and takes every wait (a warp vote);
    // lane 0 issues.  Measured on B200: 2% faster than lane 0 alone with the
    // other lanes parked at the final barrier.
    bool ok = true;
    if (n_kv > 0) {
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, err));
      };
      int nk = early_k, nv = 0;   // tiles issued
      if (lane == 0 && !closed) {
        mbar_arrive_expect_tx(&bars->q_full, TILE);
        if (VARLEN)
          tc::tma_load_3d(sQ, &tmq, 0, h, sq.q0 + s0, &bars->q_full);
        else
          tc::tma_load_2d(sQ, &tmq, 0, (b * p.nh + h) * p.S + s0, &bars->q_full);
      }
      auto load_k = [&](int t) {
        const int st = t % KS;
        if (!wait(&bars->k_empty[st], ((t / KS) & 1) ^ 1)) return false;
        nk = t + 1;
        if (t == skip || lane != 0) return true;
        mbar_arrive_expect_tx(&bars->k_full[st], TILE);
        if (VARLEN)
          tc::tma_load_3d(sK + st * TILE, &tmk, 0, j, sq.k0 + t * BKV, &bars->k_full[st]);
        else
          tc::tma_load_2d(sK + st * TILE, &tmk, 0, kv_row0 + t * BKV, &bars->k_full[st]);
        return true;
      };
      auto load_v = [&](int t) {
        const int st = t % VS;
        if (!wait(&bars->v_empty[st], ((t / VS) & 1) ^ 1)) return false;
        nv = t + 1;
        if (lane != 0) return true;
        mbar_arrive_expect_tx(&bars->v_full[st], TILE);
        if (VARLEN)
          tc::tma_load_3d(sV + st * TILE, &tmv, 0, j, sq.k0 + t * BKV, &bars->v_full[st]);
        else
          tc::tma_load_2d(sV + st * TILE, &tmv, 0, kv_row0 + t * BKV, &bars->v_full[st]);
        return true;
      };
      if (early_k == 0) {
        ok = load_k(0);
        if (ok && n_kv > 1) ok = load_k(1);
      }
      for (int t = 0; ok && t < n_kv; ++t) {
        if (t + 2 < n_kv) ok = load_k(t + 2);
        if (ok) ok = load_v(t);
      }
      // Every copy lands before the CTA may release its shared memory, also
      // when a wait gave up: wait for the last copy of each ring stage (a
      // stage's earlier copies were consumed before it was reused).  On the
      // normal path these phases have all completed already.
      if (lane == 0) {
        mbar_wait_drain(&bars->q_full, 0, err);
        for (int t = max(0, nk - KS); t < nk; ++t)
          if (t != skip) mbar_wait_drain(&bars->k_full[t % KS], (t / KS) & 1, err);
        for (int t = max(0, nv - VS); t < nv; ++t) mbar_wait_drain(&bars->v_full[t % VS], (t / VS) & 1, err);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok && sanitize) {
      const int t = n_kv - 1, st = t % VS;
      const bool landed = mbar_wait(&bars->v_full[st], (t / VS) & 1, err);
      if (__all_sync(0xffffffffu, landed)) {
        const int r0 = max(0, kv_len - t * BKV);
        uint8_t* vt = sV + st * TILE;
        for (int r = r0 + lane / 8; r < BKV; r += 4)
          *reinterpret_cast<uint4*>(vt + r * 128 + (lane % 8) * 16) = make_uint4(0, 0, 0, 0);
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
      auto issue_s = [&](int t) {   // S = Q K_t^T into the S columns
        const int ks = t % KS;
        if (!mbar_wait(&bars->k_full[ks], (t / KS) & 1, err)) return false;
        tc::fence_after_sync();
        const uint32_t k_addr = smem_u32(sK + ks * TILE);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k)
          tc::mma_bf16_ss(tmem, tc::sdesc_sw128(q_addr + k * 32, 16, 1024), tc::sdesc_sw128(k_addr + k * 32, 16, 1024),
                          IDESC_S, k != 0);
        tc::mma_commit(&bars->k_empty[ks]);
        tc::mma_commit(&bars->s_full);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int t = 0; ok && t < n_kv; ++t) {
        const int vs = t % VS;
        // S_{t+1} as soon as the softmax holds S_t in registers
        if (t + 1 < n_kv) {
          if (!mbar_wait(&bars->s_free, t & 1, err) || !issue_s(t + 1)) { ok = false; break; }
        }
        if (!mbar_wait(&bars->p_full, t & 1, err)) { ok = false; break; }
        if (!mbar_wait(&bars->v_full[vs], (t / VS) & 1, err)) { ok = false; break; }
        if (sanitize && t == n_kv - 1 && !mbar_wait(&bars->v_clean, 0, err)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t v_addr = smem_u32(sV + vs * TILE);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k)
          mma_bf16_ts(tmem + kOCol, tmem + kPCol + k * 8, tc::sdesc_sw128(v_addr + k * 2048, 16384, 1024), IDESC_O,
                      (t | k) != 0);
        tc::mma_commit(&bars->v_empty[vs]);
        tc::mma_commit(&bars->o_done);
      }
      // every MMA issued has completed before TMEM is released
      tc::mma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, err);
    }
  } else {
    // ================================================================ softmax
    const float scale_log2 = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < n_kv; ++t) {
      const int k0 = t * BKV;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, t & 1, err));
      if (!ok) break;
      tc::fence_after_sync();
      float s[BKV];
#pragma unroll
      for (int c = 0; c < BKV / 16; ++c) {
        uint32_t r[16];
        tc::tmem_ld16(tmem + lane_base + c * 16, r);
#pragma unroll
        for (int i = 0; i < 16; ++i) s[c * 16 + i] = __uint_as_float(r[i]);
      }
      tc::tmem_ld_wait();
      // S is in registers: its columns may take the next tile's scores
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free);
      const bool masked = k0 + BKV > my_lim;
      if (masked) {
#pragma unroll
        for (int i = 0; i < BKV; ++i)
          if (k0 + i >= my_lim) s[i] = -INFINITY;
      }
      // row max of the raw scores (scale > 0 commutes with max)
      float ma = -INFINITY, mb = -INFINITY, mc = -INFINITY, md = -INFINITY;
#pragma unroll
      for (int i = 0; i < BKV; i += 8) {
        ma = max3(ma, s[i], s[i + 1]);
        mb = max3(mb, s[i + 2], s[i + 3]);
        mc = max3(mc, s[i + 4], s[i + 5]);
        md = max3(md, s[i + 6], s[i + 7]);
      }
      const float mx = fmaxf(fmaxf(ma, mb), fmaxf(mc, md)) * scale_log2;
      float alpha = 1.f;
      if (m_used == -INFINITY) {
        m_used = mx;
      } else if (mx > m_used + kRescaleThreshold) {
        alpha = tc::ex2(m_used - mx);
        l *= alpha;
        m_used = mx;
      }
      // P_{t-1}.V_{t-1} has read the P columns and updated O
      if (t > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done, (t - 1) & 1, err));
        if (!ok) break;
        tc::fence_after_sync();
      }
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < HD / 16; ++c) {
          uint32_t r[16];
          tc::tmem_ld16(tmem + lane_base + kOCol + c * 16, r);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tc::tmem_st16(tmem + lane_base + kOCol + c * 16, r);
        }
      }
      // P = 2^(s * scale - m) -> bf16 pairs in the P columns
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
      // warp-uniform choice: both paths end in the .sync.aligned TMEM store
      if (kPoly > 0 && !__any_sync(0xffffffffu, masked)) {
#pragma unroll
        for (int c = 0; c < BKV / 32; ++c) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float p0 = s[c * 32 + 2 * i], p1 = s[c * 32 + 2 * i + 1];
            fma2(p0, p1, scale_log2, neg_m);
            if ((i & 7) < kPoly) {
              tc::exp2_poly2(p0, p1);
            } else {
              p0 = tc::ex2(p0);
              p1 = tc::ex2(p1);
            }
            if (i & 1) add2(sb0, sb1, p0, p1); else add2(sa0, sa1, p0, p1);
            w[i] = pack_bf16x2(p0, p1);
          }
          tc::tmem_st16(tmem + lane_base + kPCol + c * 16, w);
        }
      } else {
#pragma unroll
        for (int c = 0; c < BKV / 32; ++c) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float p0 = s[c * 32 + 2 * i], p1 = s[c * 32 + 2 * i + 1];
            fma2(p0, p1, scale_log2, neg_m);
            p0 = tc::ex2(p0);
            p1 = tc::ex2(p1);
            if (i & 1) add2(sb0, sb1, p0, p1); else add2(sa0, sa1, p0, p1);
            w[i] = pack_bf16x2(p0, p1);
          }
          tc::tmem_st16(tmem + lane_base + kPCol + c * 16, w);
        }
      }
      l += (sa0 + sa1) + (sb0 + sb1);
      tc::tmem_st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }

    if (ok && n_kv > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done, (n_kv - 1) & 1, err));
    tc::fence_after_sync();
    const size_t tok = VARLEN ? (size_t)sq.q0 + s0 + row : (size_t)b * p.S + (s0 + row);
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + (tok * p.nh + h) * HD;
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    // this warp's 32 output rows (128 bytes each) staged in the idle K ring,
    // 16-byte chunk ch of row r at chunk ch ^ (r & 7), then copied out with 8
    // lanes per row so that each store writes whole lines of 4 rows
    const uint32_t stage = smem_u32(sK) + (uint32_t)((warp & 3) * 32 * 128);
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
      uint32_t o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        o[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
      tc::st_shared_v4(stage + lane * 128 + (((2 * c) ^ (lane & 7)) << 4), o[0], o[1], o[2], o[3]);
      tc::st_shared_v4(stage + lane * 128 + (((2 * c + 1) ^ (lane & 7)) << 4), o[4], o[5], o[6], o[7]);
    }
    __syncwarp();
    {
      const unsigned long long my_dst = my_valid ? reinterpret_cast<unsigned long long>(dst) : 0ull;
      const int cc = lane & 7, rsub = lane >> 3;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = i * 4 + rsub;
        const unsigned long long d = __shfl_sync(0xffffffffu, my_dst, rr);
        uint32_t v0, v1, v2, v3;
        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v0), "=r"(v1), "=r"(v2), "=r"(v3)
                     : "r"(stage + rr * 128 + ((cc ^ (rr & 7)) << 4)) : "memory");
        if (d) tc::st_global_v4(reinterpret_cast<uint8_t*>(d) + cc * 16, v0, v1, v2, v3);
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

template <bool VARLEN>
cudaError_t launch_pair(const PrefillParams& p, cudaStream_t st) {
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = smem_attr_once(attr_set, reinterpret_cast<const void*>(prefill_pair_kernel<VARLEN>), SMEM);
      e != cudaSuccess)
    return e;
  CUtensorMap tq, tk, tv;
  if (VARLEN) {
    if (!make_tmap_packed(&tq, p.q, p.total_q, p.nh, HD)) return cudaErrorInvalidValue;
    if (!make_tmap_packed(&tk, p.k_cache, p.cap, p.nkv, HD)) return cudaErrorInvalidValue;
    if (!make_tmap_packed(&tv, p.v_cache, p.cap, p.nkv, HD)) return cudaErrorInvalidValue;
  } else {
    const uint64_t q_rows = (uint64_t)p.B * p.nh * p.S, kv_rows = (uint64_t)p.B * p.nkv * p.cap;
    if (!make_tmap_bf16_2d(&tq, p.q, HD, q_rows, HD * 2, 64, 128)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&tk, p.k_cache, HD, kv_rows, HD * 2, 64, 128)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&tv, p.v_cache, HD, kv_rows, HD * 2, 64, 128)) return cudaErrorInvalidValue;
  }
  const int n_qt = (p.S + BQ - 1) / BQ;
  const long long grid = (long long)n_qt * p.B * p.nh;
  return launch_ex(prefill_pair_kernel<VARLEN>, dim3((unsigned)grid), dim3(THREADS), SMEM, st, 1u, tq, tk, tv, p,
                   n_qt);
}

}  // namespace

cudaError_t launch_prefill_pair(const PrefillParams& p, cudaStream_t st) {
  if (p.hd != HD) return cudaErrorInvalidValue;
  return p.cu_q ? launch_pair<true>(p, st) : launch_pair<false>(p, st);
}

}  // namespace gqa
