// Split-KV decode attention on the tcgen05 tensor cores, for large head
// groups (steps a5-a6, bf16, head_dim 64 or 128, g = n_heads / n_kv_heads
// > 16: MQA and near-MQA layers).
//
// The g query heads that share a KV head read each K/V row once (MHA -> GQA
// blog, sections 3.1-3.2), so a decode step does ~g multiply-adds per cached
// byte.  On B200 the legacy mma.sync path sustains only about 1/16 of the
// tcgen05 rate, which at g = 32-48 makes the stacked-heads mma.sync kernel
// tensor-bound well below the HBM roofline.  Here the heads are the 128 rows
// of a tcgen05 tile instead: rows past g belong to other heads (or are zero
// fill) and are computed and dropped, which costs tensor time that the HBM
// stream hides.
//
// It serves large batches (the HBM-bound case); small decode steps, which are
// latency-bound, stay on the mma.sync kernel.  Measured on B200 for B 64,
// 32 heads, 1 KV head, hd 128, ragged 512..8192 keys, one call between two
// events: this kernel 51 us (42 us per call back to back), the mma.sync
// kernel 60 us, and this kernel with fixed 1024- or 2048-key splits merged
// through a workspace instead of a cluster 63 / 55 us.
// The cache is contiguous or paged: with a block table every 64-key tile is
// mapped to its page (pages hold a multiple of 64 keys, so a tile never
// crosses one), an entry outside the page pool is flagged and read as zeros.
// CTA = (sequence b, KV head j, group of <= 128 heads, key split c); the
// n_split CTAs of a (b, j, head group) form one thread-block cluster and the
// sequence's 64-key tiles are dealt out evenly over them.  Per CTA:
//   * TMEM: 256 columns = S0 | S1 (64 fp32 columns each) | O (hd).  S is
//     double-buffered: the MMA lane issues S of tile t+1 as soon as P.V of
//     tile t-1 has freed that buffer, so the tensor cores compute the next
//     scores while the softmax of tile t runs.  P is written back over the
//     first 32 columns of its S buffer as bf16 pairs and read by the P.V MMA
//     from tensor memory (A operand in TMEM).
//   * shared memory: Q (128 rows) + K/V rings of 64-key tiles (128-byte
//     swizzle); the K/V ring doubles as the merge buffer at the end.
//   * warp 0 TMA, warp 1 TMEM owner + MMA issuer, warps 2-5 softmax (thread =
//     head row; a warp whose 32 rows are all past g only keeps the barrier
//     count).  The last V tile's rows past kv_len are zeroed in shared memory
//     so that NaN padding never meets a zero probability.
// Softmax in log2 units with the lazy O rescale (only when a row max grows by
// more than 2^8).  Splits merge through distributed shared memory: each CTA
// leaves its unnormalised O rows and (m, l) in its own shared memory, and the
// cluster's threads combine them (log-sum-exp) into the bf16 output.
#include <cstddef>

#include "kernels.h"
#include "tc.cuh"

namespace gqa {
namespace {

constexpr int BM = 128, BKV = 64, THREADS = 192;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kMaxCluster = 8;
constexpr long long kMinKeys = 1ll << 18;        // B x nkv x cap below this: the mma.sync kernel

template <int HD>
struct DtCfg {
  static constexpr int KS = HD == 128 ? 2 : 3;
  static constexpr int VS = HD == 128 ? 2 : 3;
  static constexpr int NBOX = HD / 64;
  static constexpr int Q_BOX = BM * 128;                   // 128 rows x 64 columns
  static constexpr int KV_BOX = BKV * 128;                 // 64 rows x 64 columns
  static constexpr int Q_TILE = NBOX * Q_BOX;
  static constexpr int KV_TILE = NBOX * KV_BOX;
  static constexpr int Q_OFF = 0, K_OFF = Q_TILE, V_OFF = K_OFF + KS * KV_TILE, BAR_OFF = V_OFF + VS * KV_TILE;
  static constexpr int SMEM = BAR_OFF + 2048 + 1024;
  static constexpr int NCH = HD / 4;                       // float4 chunks of a partial row
  static_assert(BM * HD * 4 <= (KS + VS) * KV_TILE, "partial rows fit in the K/V ring");
  static constexpr uint32_t kOCol = 2 * BKV, kTmemCols = 256;   // S0 | S1 | O
  static constexpr uint32_t IDESC_S = tc::idesc_bf16(BM, BKV, false, false);
  static constexpr uint32_t IDESC_O = tc::idesc_bf16(BM, HD, false, true);
};

struct Bars {
  uint64_t q_full, v_clean, drain, o_done;
  uint64_t s_full[2], p_full[2];
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint32_t tmem_base;
  alignas(16) float cm[BM][2];   // per head row: m (log2 units), l; read as 8-byte pairs across the cluster
};
static_assert(offsetof(Bars, cm) % 16 == 0, "cm is read with 8-byte shared::cluster loads");
static_assert(sizeof(Bars) <= 2048, "barrier block");

template <int HD>
__global__ void __launch_bounds__(THREADS, 2)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                 const __grid_constant__ CUtensorMap tmv, DecodeParams p, int n_hg) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  using C = DtCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::BAR_OFF);
  int* err = p.err;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nsp = p.n_split;
  const int split = blockIdx.x % nsp, hg = blockIdx.x / nsp;
  const int j = blockIdx.y, b = blockIdx.z;
  const int g = p.nh / p.nkv;
  const int h0 = j * g + hg * BM;
  const int rows = min(BM, g - hg * BM);

  int kv_len = p.kv_lens[b];
  if (kv_len > p.cap || kv_len < 0) {
    if (threadIdx.x == 0 && split == 0 && hg == 0) raise_error(err, GQA_DEVERR_KVLEN_RANGE);
    kv_len = kv_len > p.cap ? p.cap : 0;
  }
  // this CTA's share of the sequence's 64-key tiles (possibly none)
  const int tiles = (kv_len + BKV - 1) / BKV;
  const int t_lo = split * tiles / nsp, t_hi = (split + 1) * tiles / nsp;
  const int n_t = t_hi - t_lo;
  const int k_lo = t_lo * BKV, k_hi = min(kv_len, t_hi * BKV);
  const bool sanitize = n_t > 0 && k_hi == kv_len && (kv_len % BKV) != 0;
  // cache row of the 64-key tile that starts at `key`: contiguous
  // [B, nkv, cap, hd], or through the block table (pages are multiples of 64
  // keys, so a tile never crosses a page); an entry outside the page pool is
  // flagged and its tile read past the pool's end, i.e. as zeros
  auto tile_row = [&](int key) {
    if (!p.block_table) return (b * p.nkv + j) * p.cap + key;
    const int lp = key / p.page_size;
    const int pg = __ldg(p.block_table + (size_t)b * p.max_pages + lp);
    if (pg < 0 || pg >= p.num_pages) {
      raise_error(err, GQA_DEVERR_PAGE_RANGE);
      return p.num_pages * p.nkv * p.page_size;
    }
    return (pg * p.nkv + j) * p.page_size + (key - lp * p.page_size);
  };

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->v_clean, 1);
    mbar_init(&bars->drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 4);
    }
    mbar_init(&bars->o_done, 1);
    for (int i = 0; i < C::KS; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < C::VS; ++i) {
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, C::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  uint8_t* sQ = smem + C::Q_OFF;
  uint8_t* sK = smem + C::K_OFF;
  uint8_t* sV = smem + C::V_OFF;
  float* part = reinterpret_cast<float*>(sK);   // merge buffer [BM][HD], reused K/V ring

  if (warp == 0) {
    // ================================================================ TMA
    bool ok = true;
    if (lane == 0 && n_t > 0) {
      mbar_arrive_expect_tx(&bars->q_full, C::Q_TILE);
      for (int bx = 0; bx < C::NBOX; ++bx)
        tc::tma_load_2d(sQ + bx * C::Q_BOX, &tmq, bx * 64, b * p.nh + h0, &bars->q_full);
      auto load_k = [&](int t) {
        const int st = t % C::KS;
        if (!mbar_wait(&bars->k_empty[st], ((t / C::KS) & 1) ^ 1, err)) return false;
        const int row = tile_row(k_lo + t * BKV);
        mbar_arrive_expect_tx(&bars->k_full[st], C::KV_TILE);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tc::tma_load_2d(sK + st * C::KV_TILE + bx * C::KV_BOX, &tmk, bx * 64, row, &bars->k_full[st]);
        return true;
      };
      auto load_v = [&](int t) {
        const int st = t % C::VS;
        if (!mbar_wait(&bars->v_empty[st], ((t / C::VS) & 1) ^ 1, err)) return false;
        const int row = tile_row(k_lo + t * BKV);
        mbar_arrive_expect_tx(&bars->v_full[st], C::KV_TILE);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tc::tma_load_2d(sV + st * C::KV_TILE + bx * C::KV_BOX, &tmv, bx * 64, row, &bars->v_full[st]);
        return true;
      };
      // K runs one tile ahead of V
      ok = load_k(0);
      for (int t = 0; ok && t < n_t; ++t) {
        if (t + 1 < n_t) ok = load_k(t + 1);
        if (ok) ok = load_v(t);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok && sanitize) {
      // zero the last V tile's rows at or past kv_len (whole 128-byte rows of every box)
      const int t = n_t - 1, st = t % C::VS;
      const bool landed = mbar_wait(&bars->v_full[st], (t / C::VS) & 1, err);
      if (__all_sync(0xffffffffu, landed)) {
        const int r0 = kv_len - (k_lo + t * BKV);
        uint8_t* vt = sV + st * C::KV_TILE;
        for (int e = r0 * 8 + lane; e < BKV * 8; e += 32)
          for (int bx = 0; bx < C::NBOX; ++bx)
            *reinterpret_cast<uint4*>(vt + bx * C::KV_BOX + e * 16) = make_uint4(0, 0, 0, 0);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->v_clean);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    if (lane == 0 && n_t > 0) {
      const uint32_t q_addr = smem_u32(sQ);
      auto issue_s = [&](int t) {   // S[t & 1] = Q K_t^T
        const int ks = t % C::KS;
        if (!mbar_wait(&bars->k_full[ks], (t / C::KS) & 1, err)) return false;
        // the buffer held P of tile t - 2: free once that tile's P.V has completed
        if (t >= 2 && !mbar_wait(&bars->o_done, (t - 2) & 1, err)) return false;
        tc::fence_after_sync();
        const uint32_t k_addr = smem_u32(sK + ks * C::KV_TILE);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k)
          tc::mma_bf16_ss(tmem + (t & 1) * BKV, tc::sdesc_sw128(q_addr + (k / 4) * C::Q_BOX + (k % 4) * 32, 16, 1024),
                          tc::sdesc_sw128(k_addr + (k / 4) * C::KV_BOX + (k % 4) * 32, 16, 1024), C::IDESC_S,
                          k != 0);
        tc::mma_commit(&bars->k_empty[ks]);
        tc::mma_commit(&bars->s_full[t & 1]);
        return true;
      };
      bool ok = mbar_wait(&bars->q_full, 0, err) && issue_s(0);
      for (int t = 0; ok && t < n_t; ++t) {
        const int vs = t % C::VS;
        if (t + 1 < n_t && !issue_s(t + 1)) break;
        if (!mbar_wait(&bars->p_full[t & 1], (t >> 1) & 1, err)) break;
        if (!mbar_wait(&bars->v_full[vs], (t / C::VS) & 1, err)) break;
        if (sanitize && t == n_t - 1 && !mbar_wait(&bars->v_clean, 0, err)) break;
        tc::fence_after_sync();
        const uint32_t v_addr = smem_u32(sV + vs * C::KV_TILE);
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k)
          tc::mma_bf16_ts(tmem + C::kOCol, tmem + (t & 1) * BKV + k * 8,
                          tc::sdesc_sw128(v_addr + k * 2048, C::KV_BOX, 1024), C::IDESC_O, (t | k) != 0);
        tc::mma_commit(&bars->v_empty[vs]);
        tc::mma_commit(&bars->o_done);
      }
      tc::mma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, err);
    }
  } else {
    // ================================================================ softmax
    const int row = (warp & 3) * 32 + lane;            // the TMEM lane quarter this warp may access
    const bool active = (warp & 3) * 32 < rows;        // warp-uniform
    const float scale_log2 = 1.4426950408889634f * rsqrtf((float)HD);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < n_t; ++t) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[t & 1], (t >> 1) & 1, err));
      if (!ok) break;
      tc::fence_after_sync();
      const uint32_t s_col = lane_base + (t & 1) * BKV;
      if (active) {
        const int k0 = k_lo + t * BKV;
        float s[BKV];
#pragma unroll
        for (int c = 0; c < BKV / 16; ++c) {
          uint32_t r[16];
          tc::tmem_ld16(tmem + s_col + c * 16, r);
#pragma unroll
          for (int i = 0; i < 16; ++i) s[c * 16 + i] = __uint_as_float(r[i]);
        }
        tc::tmem_ld_wait();
        if (k0 + BKV > k_hi) {
#pragma unroll
          for (int i = 0; i < BKV; ++i)
            if (k0 + i >= k_hi) s[i] = -INFINITY;
        }
        float ma = -INFINITY, mb = -INFINITY, mc = -INFINITY, md = -INFINITY;
#pragma unroll
        for (int i = 0; i < BKV; i += 8) {
          ma = tc::max3(ma, s[i], s[i + 1]);
          mb = tc::max3(mb, s[i + 2], s[i + 3]);
          mc = tc::max3(mc, s[i + 4], s[i + 5]);
          md = tc::max3(md, s[i + 6], s[i + 7]);
        }
        const float mx = fmaxf(fmaxf(ma, mb), fmaxf(mc, md)) * scale_log2;   // finite: key k0 is valid
        float alpha = 1.f;
        if (m_used == -INFINITY) {
          m_used = mx;
        } else if (mx > m_used + kRescaleThreshold) {
          alpha = tc::ex2(m_used - mx);
          l *= alpha;
          m_used = mx;
        }
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done, (t - 1) & 1, err));
          if (!ok) break;
          tc::fence_after_sync();
#pragma unroll
          for (int c = 0; c < HD / 16; ++c) {
            uint32_t r[16];
            tc::tmem_ld16(tmem + lane_base + C::kOCol + c * 16, r);
            tc::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tc::tmem_st16(tmem + lane_base + C::kOCol + c * 16, r);
          }
        }
        // P = 2^(s * scale - m) -> bf16 pairs over the first 32 columns of this S buffer
        const float neg_m = -m_used;
        float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
#pragma unroll
        for (int c = 0; c < BKV / 32; ++c) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float p0 = s[c * 32 + 2 * i], p1 = s[c * 32 + 2 * i + 1];
            tc::fma2(p0, p1, scale_log2, neg_m);
            p0 = tc::ex2(p0);
            p1 = tc::ex2(p1);
            if (i & 1) tc::add2(sb0, sb1, p0, p1); else tc::add2(sa0, sa1, p0, p1);
            w[i] = pack_bf16x2(p0, p1);
          }
          tc::tmem_st16(tmem + s_col + c * 16, w);
        }
        l += (sa0 + sa1) + (sb0 + sb1);
        tc::tmem_st_wait();
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[t & 1]);
    }
    // O is final once every MMA has completed, which the single-phase drain
    // barrier says (the MMA thread commits it after the last P.V).  o_done
    // cannot say it: a parity wait only tells the newest phase from the one
    // before it, and here o_done may be one phase short (P.V of the tile
    // before last still running: the last S went in ahead of it) or already
    // past both last phases.
    if (ok && n_t > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->drain, 0, err));
      // a wait that gave up anywhere (the MMA thread's included) voids O
      ok = ok && __all_sync(0xffffffffu, !(*reinterpret_cast<volatile int*>(err) & GQA_DEVERR_WAIT_TIMEOUT));
    }
    tc::fence_after_sync();
    const bool have_o = ok && n_t > 0 && active;
    if (nsp == 1) {
      // the only split: normalise and write the output rows directly
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + ((size_t)b * p.nh + h0 + row) * HD;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < HD / 16; ++c) {
        uint32_t r[16];
        if (have_o) {
          tc::tmem_ld16(tmem + lane_base + C::kOCol + c * 16, r);
          tc::tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = 0u;
        }
        if (active && row < rows) {
          uint32_t o[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            o[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
          tc::st_global_v4(dst + c * 16, o[0], o[1], o[2], o[3]);
          tc::st_global_v4(dst + c * 16 + 8, o[4], o[5], o[6], o[7]);
        }
      }
    } else if (active) {
      // this split's partial: unnormalised O rows (float4 chunk c of row r at
      // chunk c ^ (r % NCH), so that the 32 rows of a warp hit distinct banks)
      // and (m, l); a split without keys leaves m = -inf, l = 0, O = 0
#pragma unroll 1
      for (int c = 0; c < HD / 16; ++c) {
        uint32_t r[16];
        if (have_o) {
          tc::tmem_ld16(tmem + lane_base + C::kOCol + c * 16, r);
          tc::tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int ch = (c * 4 + q) ^ (row % C::NCH);
          *reinterpret_cast<uint4*>(part + row * HD + ch * 4) = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
        }
      }
      bars->cm[row][0] = have_o ? m_used : -INFINITY;
      bars->cm[row][1] = have_o ? l : 0.f;
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, C::kTmemCols);
  }
  if (nsp == 1) return;

  // ================================================================ cluster merge
  tc::cluster_sync();
  if (warp >= 2) {
    const int tid = threadIdx.x - 64;
    const uint32_t part_u = smem_u32(part), cm_u = smem_u32(&bars->cm[0][0]);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    for (int e = split * 128 + tid; e < rows * C::NCH; e += nsp * 128) {
      const int r = e / C::NCH, c = e % C::NCH;
      const int ch = c ^ (r % C::NCH);
      float2 ml[kMaxCluster];
      float M = -INFINITY;
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q) {
        if (q < nsp) {
          ml[q] = tc::ld_dsmem_f32x2(tc::mapa_shared(cm_u + r * 8, q));
          M = fmaxf(M, ml[q].x);
        }
      }
      float L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q) {
        if (q < nsp && ml[q].x != -INFINITY) {
          const float w = tc::ex2(ml[q].x - M);
          const float4 v = tc::ld_dsmem_f32x4(tc::mapa_shared(part_u + (r * HD + ch * 4) * 4, q));
          L += ml[q].y * w;
          acc.x = fmaf(v.x, w, acc.x);
          acc.y = fmaf(v.y, w, acc.y);
          acc.z = fmaf(v.z, w, acc.z);
          acc.w = fmaf(v.w, w, acc.w);
        }
      }
      const float inv = L > 0.f ? 1.f / L : 0.f;
      __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(out + ((size_t)b * p.nh + h0 + r) * HD + c * 4);
      dst[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
      dst[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    }
  }
  tc::cluster_sync();  // no CTA leaves while another may still read its shared memory
}

template <int HD>
cudaError_t launch_hd(const DecodeParams& p, int n_hg, cudaStream_t st) {
  using C = DtCfg<HD>;
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = smem_attr_once(attr_set, reinterpret_cast<const void*>(decode_tc_kernel<HD>), C::SMEM);
      e != cudaSuccess)
    return e;
  CUtensorMap tq, tk, tv;
  const uint64_t q_rows = (uint64_t)p.B * p.nh;
  const uint64_t kv_rows = p.block_table ? (uint64_t)p.num_pages * p.nkv * p.page_size : (uint64_t)p.B * p.nkv * p.cap;
  if (!make_tmap_bf16_2d(&tq, p.q, HD, q_rows, HD * 2, 64, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tk, p.k_cache, HD, kv_rows, HD * 2, 64, BKV)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tv, p.v_cache, HD, kv_rows, HD * 2, 64, BKV)) return cudaErrorInvalidValue;
  return launch_ex(decode_tc_kernel<HD>, dim3((unsigned)(p.n_split * n_hg), (unsigned)p.nkv, (unsigned)p.B),
                   dim3(THREADS), C::SMEM, st, (unsigned)p.n_split, tq, tk, tv, p, n_hg);
}

}  // namespace

// Splits per (sequence, KV head, head group) for this kernel, or 0 when a
// problem is not for it: it takes bf16 head_dim 64/128 with g > 16 and at
// least 2^18 cached key rows in all (smaller steps are latency-bound and the
// mma.sync kernel measured faster there), and caches of at most 8 x 2048 keys.
// As many splits as keep the grid within one wave of two CTAs per SM, at
// least one per 2048 keys of cache, at most one portable cluster (8).
int decode_tc_splits(const DecodeParams& p) {
  if (p.hd != 64 && p.hd != 128) return 0;
  if (p.nh / p.nkv <= 16 || (long long)p.B * p.nkv * p.cap < kMinKeys) return 0;
  const int n_hg = (p.nh / p.nkv + BM - 1) / BM;
  const long long groups = (long long)p.B * p.nkv * n_hg;
  const int by_len = (p.cap + 2047) / 2048;
  if (by_len > kMaxCluster) return 0;
  long long n = (2 * 148) / groups;
  if (n > kMaxCluster) n = kMaxCluster;
  if (n < by_len) n = by_len;
  const int tiles = (p.cap + BKV - 1) / BKV;
  if (n > tiles) n = tiles;
  return (int)(n < 1 ? 1 : n);
}

cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t st) {
  const int n_hg = (p.nh / p.nkv + BM - 1) / BM;
  if (p.n_split < 1 || p.n_split > kMaxCluster) return cudaErrorInvalidValue;
  switch (p.hd) {
    case 64: return launch_hd<64>(p, n_hg, st);
    case 128: return launch_hd<128>(p, n_hg, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gqa
