// FP8 (e4m3) prefill attention, head_dim 128, on tcgen05.mma.kind::f8f6f4
// (FlashAttention-3 summary, section "FP8低精度とincoherent processing": FP8
// doubles the tensor-core rate; the inputs come from gqa_fp8_quantize_qkv,
// whose random-sign Hadamard rotation of q and k spreads their outliers
// before rounding).  The algorithm is the exact tiled online softmax of the
// bf16 kernels (recap section; GQA head map h -> h / g, MHA -> GQA blog
// section 3.2) with both products in FP8:
//   S = Q8 K8^T            e4m3 x e4m3 -> fp32 in TMEM, times sq * sk
//   P = 2^(S' - m + 4)     rounded to e4m3 (P <= 2^8 < 448: the row max is
//                          refreshed whenever it grows by more than 2^4, and
//                          the offset 2^4 keeps probabilities down to 2^-10
//                          of the row max in e4m3's normal range)
//   O += P8 V8             e4m3 x e4m3 -> fp32 in TMEM; out = O * sv / l
// with sq, sk, sv = amax / 448 of each quantised tensor and l summed from the
// unrounded fp32 probabilities.
//
// Layout as the bf16 two-tile kernel: a CTA owns two adjacent 128-row query
// tiles of one head; TMEM S0 | S1 | O0 | O1 (4 x 128 fp32 columns), P_t
// written back over the first 32 columns of S_t (4 e4m3 per column) and fed
// to the P.V MMA from TMEM.  Tiles are 128 rows of 128 bytes (one 128-byte
// swizzle atom per row): Q and K rows of 128 features; V arrives transposed
// ([hd, keys] per KV head) so that its 128-key rows are K-major for P.V.
// 10 warps: TMA, MMA issuer, two groups of 4 softmax warps (thread = row).
#include "kernels.h"
#include "tc.cuh"

namespace gqa {
namespace {

constexpr int HD = 128, BQ = 128, BKV = 128, THREADS = 320;
constexpr int KS = 3, VS = 3;
constexpr int TILE = 128 * 128;                         // bytes
constexpr int Q_OFF = 0, K_OFF = 2 * TILE, V_OFF = K_OFF + KS * TILE, BAR_OFF = V_OFF + VS * TILE;
constexpr int SMEM = BAR_OFF + 1024 + 1024;
constexpr uint32_t O_COL = 256;
constexpr float kRescaleThreshold = 4.0f, kPOffset = 4.0f;
// Quads out of every 8 of a row chunk whose 2^x runs as a polynomial on the
// FMA pipe (tc::exp2_poly2) instead of the MUFU unit, on tiles without a
// masked key.
#ifndef GQA_FP8_POLY
#define GQA_FP8_POLY 0
#endif
constexpr int kPoly = GQA_FP8_POLY;

// Instruction descriptor, kind::f8f6f4: e4m3 A and B (format 0), f32
// accumulator (bits 4-5 = 1), both K-major, N >> 3 at bit 17, M >> 4 at 24.
constexpr uint32_t idesc_e4m3(int M, int N) { return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24); }
constexpr uint32_t IDESC = idesc_e4m3(128, 128);

__device__ __forceinline__ void mma_f8_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_f8_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n}\n"
      ::"r"(d), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// four probabilities -> one 32-bit column of e4m3 (element 0 in the low byte)
__device__ __forceinline__ uint32_t pack_e4m3x4(float p0, float p1, float p2, float p3) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(p1), "f"(p0));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(p3), "f"(p2));
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

struct Bars {
  uint64_t q_full, drain;
  uint64_t k_full[KS], k_empty[KS], v_full[VS], v_empty[VS];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint32_t tmem_base;
  int lim_max[2];
};

__global__ void __launch_bounds__(THREADS, 1)
prefill_fp8_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                   const __grid_constant__ CUtensorMap tmv, Fp8AttnParams p, int n_qt) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + BAR_OFF);
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
  const int s_base = pr * 2 * BQ;
  int kv_len = p.kv_lens[b];
  if (kv_len > p.cap || kv_len < 0) {
    if (threadIdx.x == 0) raise_error(err, GQA_DEVERR_KVLEN_RANGE);
    kv_len = kv_len > p.cap ? p.cap : 0;
  }

  const int grp = warp >= 6 ? 1 : 0;
  const int row = (warp & 3) * 32 + lane;
  int my_lim = 0;
  bool my_valid = false;
  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->drain, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < VS; ++i) {
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
    my_valid = s < p.S;
    if (my_valid) {
      const int pos = kv_len - p.S + s;
      my_lim = p.causal ? max(0, min(kv_len, pos + 1)) : kv_len;
      atomicMax(&bars->lim_max[grp], my_lim);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  const int n0 = (bars->lim_max[0] + BKV - 1) / BKV;
  const int n1 = (bars->lim_max[1] + BKV - 1) / BKV;
  const int n_kv = max(n0, n1);
  const int k_row0 = (b * p.nkv + j) * p.cap;    // K8 rows [B*nkv*cap, 128]
  const int v_row0 = (b * p.nkv + j) * HD;       // V8^T rows [B*nkv*hd, cap]
  uint8_t* sQ = smem + Q_OFF;
  uint8_t* sK = smem + K_OFF;
  uint8_t* sV = smem + V_OFF;

  if (warp == 0) {
    // ================================================================ TMA
    if (lane == 0 && n_kv > 0) {
      int nk = 0, nv = 0;
      mbar_arrive_expect_tx(&bars->q_full, 2 * TILE);
      const int qrow = (b * p.nh + h) * p.S + s_base;
      for (int t = 0; t < 2; ++t) tc::tma_load_2d(sQ + t * TILE, &tmq, 0, qrow + t * BQ, &bars->q_full);
      auto load = [&](int i, bool is_v) {
        const int S = is_v ? VS : KS;
        const int st = i % S;
        uint64_t* empty = is_v ? &bars->v_empty[st] : &bars->k_empty[st];
        uint64_t* full = is_v ? &bars->v_full[st] : &bars->k_full[st];
        if (!mbar_wait(empty, ((i / S) & 1) ^ 1, err)) return false;
        (is_v ? nv : nk) = i + 1;
        mbar_arrive_expect_tx(full, TILE);
        if (is_v)
          tc::tma_load_2d(sV + st * TILE, &tmv, i * BKV, v_row0, full);
        else
          tc::tma_load_2d(sK + st * TILE, &tmk, 0, k_row0 + i * BKV, full);
        return true;
      };
      bool ok = load(0, false);
      for (int i = 0; ok && i < n_kv; ++i) {
        if (i + 1 < n_kv) ok = load(i + 1, false);
        if (ok) ok = load(i, true);
      }
      // every copy lands before the CTA may release its shared memory
      mbar_wait_drain(&bars->q_full, 0, err);
      for (int t = max(0, nk - KS); t < nk; ++t) mbar_wait_drain(&bars->k_full[t % KS], (t / KS) & 1, err);
      for (int t = max(0, nv - VS); t < nv; ++t) mbar_wait_drain(&bars->v_full[t % VS], (t / VS) & 1, err);
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    if (lane == 0 && n_kv > 0) {
      bool ok = mbar_wait(&bars->q_full, 0, err);
      const uint32_t q_addr = smem_u32(sQ);
      const int nt[2] = {n0, n1};
      auto issue_s = [&](int t, int i) {   // S_t = Q_t K_i^T, K = 128 features in 4 steps of 32 bytes
        const uint32_t k_addr = smem_u32(sK + (i % KS) * TILE);
        const uint32_t qa = q_addr + t * TILE;
#pragma unroll
        for (int k = 0; k < HD / 32; ++k)
          mma_f8_ss(tmem + t * 128, tc::sdesc_sw128(qa + k * 32, 16, 1024), tc::sdesc_sw128(k_addr + k * 32, 16, 1024),
                    IDESC, k != 0);
        tc::mma_commit(&bars->s_full[t]);
      };
      auto issue_pv = [&](int t, int i) {  // O_t += P_t V_i, K = 128 keys in 4 steps of 32 (8 TMEM columns)
        const uint32_t v_addr = smem_u32(sV + (i % VS) * TILE);
#pragma unroll
        for (int k = 0; k < BKV / 32; ++k)
          mma_f8_ts(tmem + O_COL + t * HD, tmem + t * 128 + k * 8, tc::sdesc_sw128(v_addr + k * 32, 16, 1024), IDESC,
                    (i | k) != 0);
        tc::mma_commit(&bars->o_done[t]);
      };
      if (ok) ok = mbar_wait(&bars->k_full[0], 0, err);
      if (ok) {
        tc::fence_after_sync();
        for (int t = 0; t < 2; ++t)
          if (nt[t] > 0) issue_s(t, 0);
        tc::mma_commit(&bars->k_empty[0]);
      }
      for (int i = 0; ok && i < n_kv; ++i) {
        const int vs = i % VS, ks = (i + 1) % KS;
        ok = mbar_wait(&bars->v_full[vs], (i / VS) & 1, err);
        for (int t = 0; ok && t < 2; ++t) {
          if (i >= nt[t]) continue;
          if (!(ok = mbar_wait(&bars->p_full[t], i & 1, err))) break;
          tc::fence_after_sync();
          issue_pv(t, i);
          if (i + 1 < nt[t]) {
            if (!(ok = mbar_wait(&bars->k_full[ks], ((i + 1) / KS) & 1, err))) break;
            // S_t's columns hold P_t until P_t.V_i has completed
            if (!(ok = mbar_wait(&bars->o_done[t], i & 1, err))) break;
            tc::fence_after_sync();
            issue_s(t, i + 1);
          }
        }
        if (!ok) break;
        tc::mma_commit(&bars->v_empty[vs]);
        if (i + 1 < n_kv) tc::mma_commit(&bars->k_empty[ks]);
      }
      tc::mma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, err);
    }
  } else {
    // ================================================================ softmax (tile grp)
    // a tensor of zeros has amax 0 and codes 0; any positive scale decodes it
    // (1, as the oracle), and keeps masked scores at -inf * scale = -inf
    const float sq = p.amax[0] > 0.f ? p.amax[0] / 448.0f : 1.f;
    const float sk = p.amax[1] > 0.f ? p.amax[1] / 448.0f : 1.f;
    const float sv = p.amax[2] > 0.f ? p.amax[2] / 448.0f : 1.f;
    const float scale_log2 = 1.4426950408889634f * rsqrtf((float)HD) * sq * sk;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_col = grp * 128, o_col = O_COL + grp * HD;
    const int n_mine = grp ? n1 : n0;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < n_mine; ++i) {
      const int k0 = i * BKV;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[grp], i & 1, err));
      if (!ok) break;
      tc::fence_after_sync();
      float s[BKV];
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
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[grp], (i - 1) & 1, err));
        if (!ok) break;
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
      // P = 2^(s * scale - m + offset) -> e4m3, 4 per column, over S's first 32 columns
      const float neg_m = m_used == -INFINITY ? 0.f : kPOffset - m_used;
      float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
      const bool poly = kPoly > 0 && __all_sync(0xffffffffu, k0 + BKV <= my_lim);   // warp-uniform
#pragma unroll
      for (int c = 0; c < BKV / 64; ++c) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float p0 = s[c * 64 + 4 * e], p1 = s[c * 64 + 4 * e + 1];
          float p2 = s[c * 64 + 4 * e + 2], p3 = s[c * 64 + 4 * e + 3];
          tc::fma2(p0, p1, scale_log2, neg_m);
          tc::fma2(p2, p3, scale_log2, neg_m);
          if (poly && (e & 7) < kPoly) {
            tc::exp2_poly2(p0, p1);
            tc::exp2_poly2(p2, p3);
          } else {
            p0 = tc::ex2(p0);
            p1 = tc::ex2(p1);
            p2 = tc::ex2(p2);
            p3 = tc::ex2(p3);
          }
          tc::add2(sa0, sa1, p0, p1);
          tc::add2(sb0, sb1, p2, p3);
          w[e] = pack_e4m3x4(p0, p1, p2, p3);
        }
        tc::tmem_st16(tmem + lane_base + s_col + c * 16, w);
      }
      l += (sa0 + sa1) + (sb0 + sb1);
      tc::tmem_st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[grp]);
    }

    if (ok && n_mine > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[grp], (n_mine - 1) & 1, err));
    tc::fence_after_sync();
    const int s = s_base + grp * BQ + row;
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + (((size_t)b * p.S + s) * p.nh + h) * HD;
    const float inv_l = l > 0.f ? sv / l : 0.f;
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

}  // namespace

cudaError_t launch_prefill_fp8(const Fp8AttnParams& p, cudaStream_t st) {
  if (p.hd != HD) return cudaErrorInvalidValue;
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = smem_attr_once(attr_set, reinterpret_cast<const void*>(prefill_fp8_kernel), SMEM);
      e != cudaSuccess)
    return e;
  CUtensorMap tq, tk, tv;
  const uint64_t q_rows = (uint64_t)p.B * p.nh * p.S, k_rows = (uint64_t)p.B * p.nkv * p.cap;
  const uint64_t v_rows = (uint64_t)p.B * p.nkv * HD;
  if (!make_tmap_u8_2d(&tq, p.q8, HD, q_rows, HD, 128, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_u8_2d(&tk, p.k8, HD, k_rows, HD, 128, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_u8_2d(&tv, p.v8t, (uint64_t)p.cap, v_rows, (uint64_t)p.cap, 128, 128)) return cudaErrorInvalidValue;
  const int n_qt = (p.S + BQ - 1) / BQ;
  const long long grid = (long long)((n_qt + 1) / 2) * p.B * p.nh;
  return launch_ex(prefill_fp8_kernel, dim3((unsigned)grid), dim3(THREADS), SMEM, st, 1u, tq, tk, tv, p, n_qt);
}

}  // namespace gqa
