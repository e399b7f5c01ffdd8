// Prefill attention, two query tiles per CTA (step a4, bf16, head_dim 64/128).
//
// The algorithm is the exact tiled online softmax of the FlashAttention-3
// summary (recap section) with the GQA head map h -> h / g (MHA -> GQA blog,
// section 3.2).  The layout is Blackwell's: a CTA owns two adjacent 128-row
// query tiles of one head, which share every K/V tile.  Per tile t, TMEM holds
// S_t (128 fp32 columns; P_t is written back over its first 64 columns as
// packed bf16 pairs) and O_t (hd columns): S0 | S1 | O0 | O1 = 512 columns at
// head_dim 128.  10 warps:
//   warp 0      TMA: Q0 and Q1 once, then K and V tiles of 128 keys (K ring
//               one tile ahead of V; the last V tile's rows >= kv_len are
//               zeroed so NaN padding never meets a zero probability)
//   warp 1      allocates TMEM; one lane issues every tcgen05.mma in a
//               ping-pong order: P0.V, P1.V, then S0 = Q0.K and S1 = Q1.K of
//               the next tile, each S issued once the P.V that read its
//               columns has completed, so the tensor pipe always has the other
//               tile's work queued while a softmax group runs
//   warps 2-5   softmax of tile 0, thread = query row; warps 6-9 tile 1
// Softmax: tcgen05.ld of the S row, masking only on boundary tiles, 3-input
// max, packed f32x2 FMA for s*scale - m, ex2, packed f32x2 row sums, bf16 P
// stored back to TMEM.  O stays in TMEM and is rescaled (tcgen05.ld/st) only
// when a row's max grows by more than 2^8 (the stale max is exact after the
// final 1/l and keeps P <= 2^8).
#include "kernels.h"
#include "prefill_seq.cuh"
#include "tc.cuh"

namespace gqa {
namespace {

constexpr int BQ = 128, BKV = 128, THREADS = 320;
constexpr float kRescaleThreshold = 8.0f;
// Pairs out of every 4 whose 2^x goes to the FMA pipe (unmasked tiles).
// Measured on B200: 2 (hd 64) and 1 (hd 128) were slower than 0 - the MUFU
// unit is not what limits this kernel - so both are off.
constexpr int kPoly64 = 0, kPoly128 = 0;
// Take turns between the two softmax groups on the exponential phase (named
// barriers 2/3).  Measured on B200: no gain (the groups do not drift into
// lock-step on their own), so it is off.
constexpr bool kTurns = false;

template <int HD>
struct FaCfg {
  static constexpr int KS = HD == 128 ? 2 : 3;
  static constexpr int VS = HD == 128 ? 2 : 3;
  static constexpr int TILE = 128 * HD * 2;
  static constexpr int Q_OFF = 0;                      // Q0, Q1
  static constexpr int K_OFF = 2 * TILE;
  static constexpr int V_OFF = K_OFF + KS * TILE;
  static constexpr int BAR_OFF = V_OFF + VS * TILE;
  static constexpr int SMEM = BAR_OFF + 1024 + 1024;
  // TMEM columns.  hd 64: S0 S1 P0 P1 O0 O1 (128,128,64,64,64,64) - P has
  // its own columns, so the next S of a tile can be issued right behind its
  // P.V.  hd 128: S0 S1 O0 O1 (4 x 128) - P_t is written over S_t's first 64
  // columns, and the next S_t waits until P_t.V has completed.
  static constexpr bool P_OWN = HD == 64;
  static constexpr uint32_t P_COL = P_OWN ? 256 : 0;   // P_t at P_COL + 64 t (own) or 128 t (aliased)
  static constexpr uint32_t P_STRIDE = P_OWN ? 64 : 128;
  static constexpr uint32_t O_COL = P_OWN ? 384 : 256; // O_t at O_COL + HD t
  static constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, false, false);
  static constexpr uint32_t IDESC_O = tc::idesc_bf16(128, HD, false, true);
};

struct Bars {
  uint64_t q_full, v_clean, drain;
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint32_t tmem_base;
  int lim_max[2];
};

// VARLEN: packed variable-length sequences (3-D tensor maps over
// [tokens, heads, 64 columns]); otherwise the padded layout (2-D maps).
template <int HD, int POLY, bool VARLEN>
__global__ void __launch_bounds__(THREADS, 1)
prefill_fa_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, PrefillParams p, int n_qt) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  using C = FaCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::BAR_OFF);
  int* err = p.err;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---- work unit: a pair of query tiles, longest causal pairs first
  const int n_pairs = (n_qt + 1) / 2;
  const int bh_count = p.B * p.nh;
  const int u = blockIdx.x;
  const int pr = n_pairs - 1 - u / bh_count;
  const int b = (u % bh_count) / p.nh;
  const int h = u % p.nh;
  const int j = h / (p.nh / p.nkv);
  const int s_base = pr * 2 * BQ;   // first query row of tile 0

  const SeqRange sq = prefill_seq(p, b, err);
  if (VARLEN && s_base >= sq.S) return;   // a shorter sequence: no query in this pair (whole CTA)
  const int kv_len = sq.kv_len;

  // softmax groups: warps 2-5 -> tile 0, warps 6-9 -> tile 1
  const int grp = warp >= 6 ? 1 : 0;
  const int row = (warp & 3) * 32 + lane;
  int my_lim = 0;
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
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 4);
      mbar_init(&bars->o_done[t], 1);
      bars->lim_max[t] = 0;
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, 512);
  __syncthreads();
  if (warp >= 2) {
    const int s = s_base + grp * BQ + row;
    my_valid = s < sq.S;
    if (my_valid) {
      const int pos = p.q_pos ? p.q_pos[(size_t)b * p.S + s] : kv_len - sq.S + s;
      my_lim = p.causal ? max(0, min(kv_len, pos + 1)) : kv_len;
      atomicMax(&bars->lim_max[grp], my_lim);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  const int n0 = (bars->lim_max[0] + BKV - 1) / BKV;   // KV tiles each query tile needs
  const int n1 = (bars->lim_max[1] + BKV - 1) / BKV;
  const int n_kv = max(n0, n1);
  const bool sanitize = n_kv > 0 && kv_len < n_kv * BKV;
  const int kv_row0 = VARLEN ? 0 : (b * p.nkv + j) * p.cap;
  uint8_t* sQ = smem + C::Q_OFF;
  uint8_t* sK = smem + C::K_OFF;
  uint8_t* sV = smem + C::V_OFF;

  if (warp == 0) {
    // ================================================================ TMA
    bool ok = true;
    if (lane == 0 && n_kv > 0) {
      mbar_arrive_expect_tx(&bars->q_full, 2 * C::TILE);
      const int qrow = VARLEN ? 0 : (b * p.nh + h) * p.S + s_base;
      for (int t = 0; t < 2; ++t)
        for (int c = 0; c < HD / 64; ++c) {
          if (VARLEN)
            tc::tma_load_3d(sQ + t * C::TILE + c * 16384, &tmq, c * 64, h, sq.q0 + s_base + t * BQ, &bars->q_full);
          else
            tc::tma_load_2d(sQ + t * C::TILE + c * 16384, &tmq, c * 64, qrow + t * BQ, &bars->q_full);
        }
      auto load = [&](int i, bool is_v) {
        const int S = is_v ? C::VS : C::KS;
        const int st = i % S;
        uint64_t* empty = is_v ? &bars->v_empty[st] : &bars->k_empty[st];
        uint64_t* full = is_v ? &bars->v_full[st] : &bars->k_full[st];
        if (!mbar_wait(empty, ((i / S) & 1) ^ 1, err)) return false;
        mbar_arrive_expect_tx(full, C::TILE);
        uint8_t* dst = (is_v ? sV : sK) + st * C::TILE;
        for (int c = 0; c < HD / 64; ++c) {
          if (VARLEN)
            tc::tma_load_3d(dst + c * 16384, is_v ? &tmv : &tmk, c * 64, j, sq.k0 + i * BKV, full);
          else
            tc::tma_load_2d(dst + c * 16384, is_v ? &tmv : &tmk, c * 64, kv_row0 + i * BKV, full);
        }
        return true;
      };
      ok = load(0, false);
      for (int i = 0; ok && i < n_kv; ++i) {
        if (i + 1 < n_kv) ok = load(i + 1, false);
        if (ok) ok = load(i, true);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok && sanitize) {
      const int t = n_kv - 1, st = t % C::VS;
      const bool landed = mbar_wait(&bars->v_full[st], (t / C::VS) & 1, err);
      if (__all_sync(0xffffffffu, landed)) {
        const int r0 = max(0, kv_len - t * BKV);
        uint8_t* vt = sV + st * C::TILE;
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
      const int nt[2] = {n0, n1};
      auto issue_s = [&](int t, int i) {   // S_t = Q_t K_i^T
        const uint32_t k_addr = smem_u32(sK + (i % C::KS) * C::TILE);
        const uint32_t qa = q_addr + t * C::TILE;
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (k / 4) * 16384 + (k % 4) * 32;
          tc::mma_bf16_ss(tmem + t * 128, tc::sdesc_sw128(qa + off, 16, 1024), tc::sdesc_sw128(k_addr + off, 16, 1024),
                          C::IDESC_S, k != 0);
        }
        tc::mma_commit(&bars->s_full[t]);
      };
      auto issue_pv = [&](int t, int i) {  // O_t += P_t V_i
        const uint32_t v_addr = smem_u32(sV + (i % C::VS) * C::TILE);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k)
          tc::mma_bf16_ts(tmem + C::O_COL + t * HD, tmem + C::P_COL + t * C::P_STRIDE + k * 8,
                          tc::sdesc_sw128(v_addr + k * 2048, 16384, 1024), C::IDESC_O, (i | k) != 0);
        tc::mma_commit(&bars->o_done[t]);
      };
      if (ok) ok = mbar_wait(&bars->k_full[0], 0, err);
      if (ok) {
        tc::fence_after_sync();
        for (int t = 0; t < 2; ++t)
          if (nt[t] > 0) issue_s(t, 0);
        tc::mma_commit(&bars->k_empty[0]);
      }
      // ping-pong: P0.V_i, S0 of tile i+1, P1.V_i, S1 of tile i+1, ...
      for (int i = 0; ok && i < n_kv; ++i) {
        const int vs = i % C::VS, ks = (i + 1) % C::KS;
        ok = mbar_wait(&bars->v_full[vs], (i / C::VS) & 1, err);
        if (ok && sanitize && i == n_kv - 1) ok = mbar_wait(&bars->v_clean, 0, err);
        for (int t = 0; ok && t < 2; ++t) {
          if (i >= nt[t]) continue;
          if (!(ok = mbar_wait(&bars->p_full[t], i & 1, err))) break;
          tc::fence_after_sync();
          issue_pv(t, i);
          if (i + 1 < nt[t]) {
            if (!(ok = mbar_wait(&bars->k_full[ks], ((i + 1) / C::KS) & 1, err))) break;
            // aliased P: S_t's columns hold P_t until P_t.V_i has completed
            if (!C::P_OWN && !(ok = mbar_wait(&bars->o_done[t], i & 1, err))) break;
            tc::fence_after_sync();
            issue_s(t, i + 1);
          }
        }
        if (!ok) break;
        tc::mma_commit(&bars->v_empty[vs]);
        if (i + 1 < n_kv) tc::mma_commit(&bars->k_empty[ks]);
      }
      tc::mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, err);
    }
  } else {
    // ================================================================ softmax (tile grp)
    const float scale_log2 = 1.4426950408889634f * rsqrtf((float)HD);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_col = grp * 128, p_col = C::P_COL + grp * C::P_STRIDE, o_col = C::O_COL + grp * HD;
    const int n_mine = grp ? n1 : n0;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    // The two groups take turns on the exponential phase: a token passed
    // through named barriers 2 (group 0's turn) and 3 (group 1's turn), so
    // that one group's MUFU work overlaps the other group's MMAs instead of
    // both exponentiating at once (they would drift into lock-step).  Both
    // groups run the same n_kv rounds and never leave the loop early, so
    // every barrier arrival is matched even when a wait gives up.
    const int rounds = n_kv;
    const int my_bar = 2 + grp, other_bar = 3 - grp;
    if (kTurns && grp == 1 && rounds > 0) tc::named_arrive(2, 256);   // group 0 goes first
    for (int i = 0; i < rounds; ++i) {
      const int k0 = i * BKV;
      bool work = ok && i < n_mine;   // warp-uniform
      if (work) work = ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[grp], i & 1, err));
      float s[BKV];
      if (work) {
      tc::fence_after_sync();
#pragma unroll
      for (int c = 0; c < BKV / 16; ++c) {
        uint32_t r[16];
        tc::tmem_ld16(tmem + lane_base + s_col + c * 16, r);
#pragma unroll
        for (int e = 0; e < 16; ++e) s[c * 16 + e] = __uint_as_float(r[e]);
      }
      tc::tmem_ld_wait();
      if (k0 + BKV > my_lim) {
#pragma unroll
        for (int e = 0; e < BKV; ++e)
          if (k0 + e >= my_lim) s[e] = -INFINITY;
      }
      float ma = -INFINITY, mb = -INFINITY, mc = -INFINITY, md = -INFINITY;
#pragma unroll
      for (int e = 0; e < BKV; e += 8) {
        ma = tc::max3(ma, s[e], s[e + 1]);
        mb = tc::max3(mb, s[e + 2], s[e + 3]);
        mc = tc::max3(mc, s[e + 4], s[e + 5]);
        md = tc::max3(md, s[e + 6], s[e + 7]);
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
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
        // O_t must hold P_t.V_{i-1} before it is scaled
        work = ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[grp], (i - 1) & 1, err));
        if (work) {
          tc::fence_after_sync();
#pragma unroll
          for (int c = 0; c < HD / 16; ++c) {
            uint32_t r[16];
            tc::tmem_ld16(tmem + lane_base + o_col + c * 16, r);
            tc::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tc::tmem_st16(tmem + lane_base + o_col + c * 16, r);
          }
        }
      }
      // own P columns: free once P_t.V_{i-1} has read them
      if (C::P_OWN && i > 0 && work)
        work = ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[grp], (i - 1) & 1, err));
      }  // work: S loaded, max and rescale done
      if (kTurns) tc::named_sync(my_bar, 256);    // take the token
      if (work) {
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
      // warp-uniform choice: both paths end in the .sync.aligned TMEM store
      if (__all_sync(0xffffffffu, k0 + BKV <= my_lim)) {
        // no masked key in the warp: POLY of every 4 pairs take 2^x on the FMA pipe
#pragma unroll
        for (int c = 0; c < BKV / 32; ++c) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float p0 = s[c * 32 + 2 * e], p1 = s[c * 32 + 2 * e + 1];
            tc::fma2(p0, p1, scale_log2, neg_m);
            if ((e & 3) < POLY) {
              tc::exp2_poly2(p0, p1);
            } else {
              p0 = tc::ex2(p0);
              p1 = tc::ex2(p1);
            }
            if (e & 1) tc::add2(sb0, sb1, p0, p1); else tc::add2(sa0, sa1, p0, p1);
            w[e] = pack_bf16x2(p0, p1);
          }
          tc::tmem_st16(tmem + lane_base + p_col + c * 16, w);
        }
      } else {
#pragma unroll
        for (int c = 0; c < BKV / 32; ++c) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float p0 = s[c * 32 + 2 * e], p1 = s[c * 32 + 2 * e + 1];
            tc::fma2(p0, p1, scale_log2, neg_m);
            p0 = tc::ex2(p0);
            p1 = tc::ex2(p1);
            if (e & 1) tc::add2(sb0, sb1, p0, p1); else tc::add2(sa0, sa1, p0, p1);
            w[e] = pack_bf16x2(p0, p1);
          }
          tc::tmem_st16(tmem + lane_base + p_col + c * 16, w);
        }
      }
      l += (sa0 + sa1) + (sb0 + sb1);
      }  // work
      // pass the token (group 1's last arrival would have no matching wait)
      if (kTurns && (grp == 0 || i + 1 < rounds)) tc::named_arrive(other_bar, 256);
      if (work) {
        tc::tmem_st_wait();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[grp]);
      }
    }

    if (ok && n_mine > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[grp], (n_mine - 1) & 1, err));
    tc::fence_after_sync();
    const int s = s_base + grp * BQ + row;
    const size_t tok = VARLEN ? (size_t)sq.q0 + s : (size_t)b * p.S + s;
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + (tok * p.nh + h) * HD;
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
    for (int c = 0; c < HD / 16; ++c) {
      uint32_t r[16];
      if (ok && n_mine > 0) {
        __syncwarp();
        tc::tmem_ld16(tmem + lane_base + o_col + c * 16, r);
        tc::tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = 0u;
      }
      if (my_valid) {
        uint32_t o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          o[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
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
    tc::tmem_dealloc(tmem, 512);
  }
}

template <int HD, int POLY, bool VARLEN>
cudaError_t launch_hd(const PrefillParams& p, cudaStream_t st) {
  using C = FaCfg<HD>;
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = smem_attr_once(attr_set, reinterpret_cast<const void*>(prefill_fa_kernel<HD, POLY, VARLEN>),
                                     C::SMEM);
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
  const long long grid = (long long)((n_qt + 1) / 2) * p.B * p.nh;
  return launch_ex(prefill_fa_kernel<HD, POLY, VARLEN>, dim3((unsigned)grid), dim3(THREADS), C::SMEM, st, 1u, tq, tk,
                   tv, p, n_qt);
}

}  // namespace

cudaError_t launch_prefill_fa(const PrefillParams& p, cudaStream_t st) {
  const bool packed = p.cu_q != nullptr;
  switch (p.hd) {
    case 64: return packed ? launch_hd<64, kPoly64, true>(p, st) : launch_hd<64, kPoly64, false>(p, st);
    case 128: return packed ? launch_hd<128, kPoly128, true>(p, st) : launch_hd<128, kPoly128, false>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gqa
