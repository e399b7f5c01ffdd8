// Split-KV decode attention for large head groups on the tcgen05 tensor
// cores, with the keys as the MMA rows (steps a5-a6; bf16, head_dim 128,
// 16 < g <= 64 query heads per KV head: MQA and near-MQA layers).
//
// The g query heads that share a KV head read each K/V row once (MHA -> GQA
// blog, sections 3.1-3.2).  One 128-key tile of K is the M = 128 side of the
// score MMA and the g heads (padded to NP, a multiple of 16) are its N side:
//   S^T[key, h] = K_tile . Q^T           M 128 keys, N NP heads, K 128 dims
//   O^T[d, h]  += V_tile^T . P^T         M 128 dims, N NP heads, K 128 keys
// so no MMA row is wasted (stacking the g heads as the 128 rows wastes
// 128 - g of them).  P^T goes through shared memory as the K-major B operand
// (one row of 128 keys per head); V^T is the MN-major A operand, read
// straight from the TMA tile.
//
// Work split: the 128-key tiles of all (sequence, KV head) units are laid
// end to end and cut into one equal range per CTA, one CTA per SM, so every
// SM streams the same number of K/V bytes whatever the length mix.  A range
// holds pieces of one or more units.  A piece that is a whole unit writes its
// output directly; the other pieces leave a partial (o unnormalised, m, l) in
// the workspace and the last piece of a unit to finish merges them (counter).
//
// Warps: 0 TMA (Q per piece; K and V tiles as 64-key boxes, so that a paged
// cache maps each half tile to its page), 1 TMEM owner + MMA issuer, 2-5
// softmax (thread = key of the tile), 6-9 epilogue (thread = head dimension).
// TMEM: S^T double-buffered (2 x NP columns); O^T double-buffered across
// pieces, so the epilogue of a piece overlaps the next piece.  Each O^T
// buffer has NP more columns for the softmax denominators: a second MMA per
// tile multiplies P^T by an all-ones A operand held in TMEM, so that every
// row of those columns accumulates l_h = sum over keys of P[h][key] (from the
// same bf16 P as the numerator), rescaled together with O^T.
// Softmax in log2 units with a lazy maximum per head: a tile whose scores stay
// within 2^8 of the running maxima is exponentiated against them unchanged;
// otherwise the CTA takes the exact column maxima (transposed warp
// reductions, then across the four warps) and rescales O^T with its
// denominators.  Rows past kv_len in the unit's last V tile are zeroed in
// shared memory by the softmax threads that own those keys, so NaN padding
// never meets a zero probability.
// Shared memory: K and V rings of 128-key tiles (32 KB a stage; 3 + 3 stages
// for up to 32 heads), Q double-buffered across pieces, one P^T buffer (the
// softmax writes P(n) once P.V(n-1) has completed, which also frees O^T for
// a rescale).  K/V are loaded evict-first in L2, so the partials a merge
// reads back stay resident.  A merge by a CTA's last piece brings the
// partials into the then idle K/V ring with one bulk copy each; other merges
// read them in rounds of two pieces from the workspace.
// Measured on B200 for the B 64 MQA decode (32 heads, ragged 512..8192 keys,
// 167 MB of K/V): ~1.5-1.9 us per tile and SM while streaming, ~7 us of
// launch, prefix sums and first-tile latency, ~4-6 us of partial epilogues
// and final merges.  That is slower than the cluster kernel on caches of up
// to 8 x 2048 keys, contiguous or paged (51 against 42 us when the calls run
// back to back), so the dispatcher uses this kernel for longer caches only.
#include <atomic>
#include <cstddef>

#include "kernels.h"
#include "tc.cuh"

namespace gqa {
namespace {

constexpr int HD = 128, BKEY = 128, THREADS = 320;
constexpr int kMaxUnits = 512;                 // (sequence, KV head) units: tile prefix sums in shared memory
constexpr int kMaxGrid = kHnMaxGrid;
constexpr float kRescaleThreshold = 8.0f;
constexpr long long kMinKeys = 1ll << 18;      // B x nkv x cap below this: latency-bound, the mma.sync kernel

// Ring depths.  Under full load a K/V copy takes ~4 us to land on B200, about
// three times the ~1.4 us in which one SM streams a 64 KB tile at its share of
// HBM bandwidth, and a ring slot is reused only once its tile is consumed, so
// each ring needs 3 slots to keep the stream at bandwidth.  3 + 3 slots of
// 32 KB fit next to Q and P for 32 heads; 48 and 64 heads give up one slot.
template <int NP>
struct HnCfg {
  static constexpr int KS = NP == 48 ? 2 : 3, VS = NP == 64 ? 2 : 3;
  static constexpr int BOX = 64 * 128;                 // 64 rows x 128 bytes
  static constexpr int KV_TILE = 4 * BOX;              // 128 keys x 128 dims
  static constexpr int Q_BOX = NP * 128, Q_TILE = 2 * Q_BOX;
  static constexpr int P_BOX = NP * 128, P_TILE = 2 * P_BOX;
  static constexpr int K_OFF = 0, V_OFF = KS * KV_TILE, Q_OFF = V_OFF + VS * KV_TILE;
  static constexpr int P_OFF = Q_OFF + 2 * Q_TILE, BAR_OFF = P_OFF + P_TILE;
  // TMEM columns: S^T 0 | S^T 1 | O^T 0, L 0 | O^T 1, L 1 | ones
  static constexpr uint32_t S_COL = 0, O_COL = 2 * NP, ONES_COL = 6 * NP;
  static constexpr uint32_t TMEM_COLS = 6 * NP + 8 <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_S = tc::idesc_bf16(128, NP, false, false);
  static constexpr uint32_t IDESC_O = tc::idesc_bf16(128, NP, true, false);
  static_assert(NP % 16 == 0 && NP >= 32 && NP <= 64, "heads as N");
};

template <int NP>
struct Bars {
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t q_full[2], q_empty[2], s_full[2], s_free[2], p_full, p_empty;
  uint64_t o_final[2], o_empty[2], ml_full[2], ml_empty[2], drain, merge_full;
  uint32_t tmem_base;
  unsigned last;
  alignas(16) float m_used[NP];          // running maximum per head (log2 units) of the current piece
  alignas(16) float alpha[NP];           // rescale factors of the current tile
  float red[4][NP];                      // per-warp column reductions of the softmax warps
  float mh[2][NP];                       // per piece parity: m per head, softmax -> epilogue
  int prefix[kMaxUnits + 1];             // exclusive prefix sums of tiles per unit
  int lens[kMaxUnits];                   // kv_len per sequence, clamped to [0, cap]
  int warp_tot[THREADS / 32];
};

template <int NP>
constexpr int hn_smem_bytes() {
  return HnCfg<NP>::BAR_OFF + (int)sizeof(Bars<NP>) + 1024;
}

__device__ __forceinline__ int clamp_len(int v, int cap) { return v > cap ? cap : (v < 0 ? 0 : v); }

// OR of a predicate over the `n` threads of named barrier `id` (a barrier too)
__device__ __forceinline__ bool named_any(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r) : "r"((uint32_t)v), "r"(id), "r"(n) : "memory");
  return r != 0;
}

__device__ __forceinline__ void st_shared_u16(uint32_t a, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(v) : "memory");
}

// Transposed warp reduction: lane i holds 32 values v[0..31]; afterwards v[0]
// of lane i is the max (or sum) over all lanes of index i.  Each step halves
// the values a lane keeps (the half whose index bit matches the lane's bit)
// and folds in the partner's copy of that half: 31 shuffles for 32 columns.
template <bool MAX>
__device__ __forceinline__ float transpose_reduce32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = upper ? v[i] : v[i + o];
      const float keep = upper ? v[i + o] : v[i];
      const float r = __shfl_xor_sync(0xffffffffu, send, o);
      v[i] = MAX ? fmaxf(keep, r) : keep + r;
    }
  }
  return v[0];
}

// per-warp column reduction of s[0..NP) into red[q][.]
template <int NP, bool MAX>
__device__ __forceinline__ void warp_columns(const float (&s)[NP], float* red_q) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int grp = 0; grp < (NP + 31) / 32; ++grp) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = grp * 32 + i < NP ? s[grp * 32 + i] : (MAX ? -INFINITY : 0.f);
    const float r = transpose_reduce32<MAX>(v);
    if (grp * 32 + lane < NP) red_q[grp * 32 + lane] = r;
  }
}

// first unit u with prefix[u] <= x < prefix[u + 1] (x < prefix[U])
__device__ __forceinline__ int unit_of(const int* prefix, int U, int x) {
  int lo = 1, hi = U;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] > x) hi = mid; else lo = mid + 1;
  }
  return lo - 1;
}

// The CTA whose range [c*T/G, (c+1)*T/G) holds global tile x.
__device__ __forceinline__ int cta_of(long long x, long long T, int G) { return (int)(((x + 1) * G - 1) / T); }

// Walks the pieces of this CTA's tile range in order: unit u, tiles [t_lo, t_hi).
struct PieceWalk {
  const int* prefix;
  int U, x, end;
  int u, t_lo, t_hi;
  __device__ bool next() {
    if (x >= end) return false;
    u = unit_of(prefix, U, x);
    t_lo = x - prefix[u];
    t_hi = min(end, prefix[u + 1]) - prefix[u];
    x = prefix[u] + t_hi;
    return true;
  }
};

// One step of the log-sum-exp merge: fold a piece's (m, l, o) into the
// running (M, L, acc).  Both merges below take exactly these steps, in piece
// order, with every product rounded on its own (no contraction into an FMA
// the compiler might choose differently in the two places), so that a unit's
// output has the same bits whichever of its pieces finishes last and merges.
__device__ __forceinline__ void merge_step(float& M, float& L, float4& acc, float m_k, float l_k, const float4& v) {
  if (m_k == -INFINITY) return;
  const float Mn = fmaxf(M, m_k);
  const float a = tc::ex2(M - Mn), wk = tc::ex2(m_k - Mn);
  L = fmaf(l_k, wk, __fmul_rn(L, a));
  acc.x = fmaf(v.x, wk, __fmul_rn(acc.x, a));
  acc.y = fmaf(v.y, wk, __fmul_rn(acc.y, a));
  acc.z = fmaf(v.z, wk, __fmul_rn(acc.z, a));
  acc.w = fmaf(v.w, wk, __fmul_rn(acc.w, a));
  M = Mn;
}

__device__ __forceinline__ void merge_store(__nv_bfloat16* dst_row, int d4, float L, const float4& acc) {
  const float inv = L > 0.f ? 1.f / L : 0.f;
  __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(dst_row + d4);
  dst[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  dst[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
}

// Merge of a unit's np partials, written to workspace slots slot0 .. slot0 +
// np - 1 (o rows, then (m, l) per head), into its bf16 output rows, by the 128
// epilogue threads (te).  Per group of 32 heads, thread te takes float4
// columns d4 of heads hg + h0, hg + h0 + 4, ...; the pieces go two at a time
// with all their (m, l) and o loads in flight at once.  Kept out of line so
// that its registers do not add to those of the pipeline loops.
template <int NP>
__device__ __noinline__ void merge_unit(const DecodeParams& p, int g, int b, int j, int slot0, int np, int te,
                                        __nv_bfloat16* out) {
  constexpr int WS_ROW = HD + kWsPad;
  constexpr int NH = 8;                          // heads per thread and group
  constexpr int KC = 2;                          // pieces per round of loads
  const int d4 = (te & 31) * 4, h0 = te >> 5;
#pragma unroll 1
  for (int hg = 0; hg < g; hg += 32) {
    float M[NH], Lr[NH];
    float4 acc[NH];
#pragma unroll
    for (int i = 0; i < NH; ++i) {
      M[i] = -INFINITY;
      Lr[i] = 0.f;
      acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll 1
    for (int k0 = 0; k0 < np; k0 += KC) {
      float2 ml[KC][NH];
      float4 ov[KC][NH];
#pragma unroll
      for (int k = 0; k < KC; ++k) {
        const float* slot_k = p.ws + (size_t)(slot0 + k0 + k) * NP * WS_ROW;
#pragma unroll
        for (int i = 0; i < NH; ++i) {
          const int h = hg + h0 + 4 * i;
          if (k0 + k < np && h < g) {
            ml[k][i] = __ldcg(reinterpret_cast<const float2*>(slot_k + h * WS_ROW + HD));
            ov[k][i] = __ldcg(reinterpret_cast<const float4*>(slot_k + h * WS_ROW + d4));
          } else {
            ml[k][i] = make_float2(-INFINITY, 0.f);
            ov[k][i] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      }
#pragma unroll
      for (int k = 0; k < KC; ++k)
#pragma unroll
        for (int i = 0; i < NH; ++i) merge_step(M[i], Lr[i], acc[i], ml[k][i].x, ml[k][i].y, ov[k][i]);
    }
#pragma unroll
    for (int i = 0; i < NH; ++i) {
      const int h = hg + h0 + 4 * i;
      if (h < g) merge_store(out + ((size_t)b * p.nh + j * g + h) * HD, d4, Lr[i], acc[i]);
    }
  }
}

// The same merge from np partials already in shared memory (`part`, slot k at
// k * NP * (HD + kWsPad) floats): thread te takes float4 columns d4 of heads
// h0, h0 + 4, ...; (m, l) are read as broadcasts.
template <int NP>
__device__ __noinline__ void merge_smem(const float* part, const DecodeParams& p, int g, int b, int j, int np,
                                           int te, __nv_bfloat16* out) {
  constexpr int WS_ROW = HD + kWsPad;
  const int d4 = (te & 31) * 4, h0 = te >> 5;
#pragma unroll 2
  for (int h = h0; h < g; h += 4) {
    float M = -INFINITY, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < np; ++k) {
      const float* row = part + ((size_t)k * NP + h) * WS_ROW;
      merge_step(M, L, acc, row[HD], row[HD + 1], *reinterpret_cast<const float4*>(row + d4));
    }
    merge_store(out + ((size_t)b * p.nh + j * g + h) * HD, d4, L, acc);
  }
}

template <int NP>
__global__ void __launch_bounds__(THREADS, 1)
decode_hn_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                 const __grid_constant__ CUtensorMap tmv, DecodeParams p, int rows_total) {
  pdl_launch_dependents();
  pdl_wait();   // inputs may come from the kernel before this one
  using C = HnCfg<NP>;
  constexpr int KS = C::KS, VS = C::VS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars<NP>* bars = reinterpret_cast<Bars<NP>*>(smem + C::BAR_OFF);
  uint8_t* sK = smem + C::K_OFF;
  uint8_t* sV = smem + C::V_OFF;
  uint8_t* sQ = smem + C::Q_OFF;
  uint8_t* sP = smem + C::P_OFF;
  int* err = p.err;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = p.nh / p.nkv;
  const int U = p.B * p.nkv;

  if (threadIdx.x == 0) {
    for (int i = 0; i < KS; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 1);
      mbar_init(&bars->q_empty[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 4);
      mbar_init(&bars->o_final[i], 1);
      mbar_init(&bars->o_empty[i], 4);
      mbar_init(&bars->ml_full[i], 1);
      mbar_init(&bars->ml_empty[i], 4);
    }
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->p_empty, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->merge_full, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < NP) bars->m_used[threadIdx.x] = -INFINITY;
  if (threadIdx.x == 32) {   // the tensor-map fetches overlap the prefix sums below
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, C::TMEM_COLS);

  // ---- tiles per unit -> exclusive prefix sums (every thread takes a chunk)
  {
    const int per = (U + THREADS - 1) / THREADS;
    const int u0 = threadIdx.x * per;
    int sum = 0;
    for (int k = 0; k < per; ++k) {
      const int u = u0 + k;
      if (u < U) {
        const int b = u / p.nkv;
        const int raw = p.kv_lens[b];
        if (u % p.nkv == 0) {
          if ((raw > p.cap || raw < 0) && blockIdx.x == 0) raise_error(err, GQA_DEVERR_KVLEN_RANGE);
          bars->lens[b] = clamp_len(raw, p.cap);
        }
        sum += (clamp_len(raw, p.cap) + BKEY - 1) / BKEY;
      }
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) bars->warp_tot[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += bars->warp_tot[w];
    base += incl - sum;
    for (int k = 0; k < per; ++k) {
      const int u = u0 + k;
      if (u < U) {
        bars->prefix[u] = base;
        base += (clamp_len(p.kv_lens[u / p.nkv], p.cap) + BKEY - 1) / BKEY;
        if (u == U - 1) bars->prefix[U] = base;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  // The tiles are cut over G = min(grid, tiles) CTAs, so that every range
  // holds at least one tile and the pieces of a unit sit on consecutive CTAs
  // (a merge counts them as c_last - c_first + 1); CTAs past G idle.
  const long long T = bars->prefix[U];
  const int G = T < (long long)gridDim.x ? (T > 0 ? (int)T : 1) : (int)gridDim.x;
  const int c_me = (int)blockIdx.x;
  const int r_begin = c_me < G ? (int)((long long)c_me * T / G) : (int)T;
  const int r_end = c_me < G ? (int)((long long)(c_me + 1) * T / G) : (int)T;

  if (warp == 0) {
    // ================================================================ TMA
    if (lane == 0) {
      // cache row of a 64-key box: contiguous [B, nkv, cap, hd] or through the
      // block table; a box wholly past kv_len (or with a page outside the
      // pool) points past the end of the tensor map, which reads zeros
      auto box_row = [&](int b, int j, int key, int kv_len) -> int {
        if (key >= kv_len) return rows_total;
        if (!p.block_table) return (b * p.nkv + j) * p.cap + key;
        const int lp = key / p.page_size;
        const int pg = __ldg(p.block_table + (size_t)b * p.max_pages + lp);
        if (pg < 0 || pg >= p.num_pages) {
          raise_error(err, GQA_DEVERR_PAGE_RANGE);
          return rows_total;
        }
        return (pg * p.nkv + j) * p.page_size + (key - lp * p.page_size);
      };
      // K/V are read once: evict-first in L2, so that the partials the merges
      // read back stay resident
      const uint64_t stream_policy = tc::l2_policy_evict_first();
      int nk = 0, nv = 0, nq = 0;
      int pend_r0 = 0, pend_r1 = 0;
      auto load_v = [&](int r0, int r1) {
        const int st = nv % VS;
        if (!mbar_wait(&bars->v_empty[st], ((nv / VS) & 1) ^ 1, err)) return false;
        mbar_arrive_expect_tx(&bars->v_full[st], C::KV_TILE);
        uint8_t* dst = sV + st * C::KV_TILE;   // boxes [key half][dim half]
        tc::tma_load_2d_hint(dst, &tmv, 0, r0, &bars->v_full[st], stream_policy);
        tc::tma_load_2d_hint(dst + C::BOX, &tmv, 64, r0, &bars->v_full[st], stream_policy);
        tc::tma_load_2d_hint(dst + 2 * C::BOX, &tmv, 0, r1, &bars->v_full[st], stream_policy);
        tc::tma_load_2d_hint(dst + 3 * C::BOX, &tmv, 64, r1, &bars->v_full[st], stream_policy);
        ++nv;
        return true;
      };
      bool ok = true;
      PieceWalk w{bars->prefix, U, r_begin, r_end};
      while (ok && w.next()) {
        const int b = w.u / p.nkv, j = w.u % p.nkv;
        const int kv_len = bars->lens[b];
        const int qb = nq & 1;
        if (!mbar_wait(&bars->q_empty[qb], ((nq >> 1) & 1) ^ 1, err)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars->q_full[qb], C::Q_TILE);
        tc::tma_load_2d(sQ + qb * C::Q_TILE, &tmq, 0, b * p.nh + j * g, &bars->q_full[qb]);
        tc::tma_load_2d(sQ + qb * C::Q_TILE + C::Q_BOX, &tmq, 64, b * p.nh + j * g, &bars->q_full[qb]);
        ++nq;
        for (int t = w.t_lo; t < w.t_hi; ++t) {
          const int r0 = box_row(b, j, t * BKEY, kv_len), r1 = box_row(b, j, t * BKEY + 64, kv_len);
          const int st = nk % KS;
          if (!mbar_wait(&bars->k_empty[st], ((nk / KS) & 1) ^ 1, err)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars->k_full[st], C::KV_TILE);
          uint8_t* dst = sK + st * C::KV_TILE;   // boxes [dim half][key half]
          tc::tma_load_2d_hint(dst, &tmk, 0, r0, &bars->k_full[st], stream_policy);
          tc::tma_load_2d_hint(dst + C::BOX, &tmk, 0, r1, &bars->k_full[st], stream_policy);
          tc::tma_load_2d_hint(dst + 2 * C::BOX, &tmk, 64, r0, &bars->k_full[st], stream_policy);
          tc::tma_load_2d_hint(dst + 3 * C::BOX, &tmk, 64, r1, &bars->k_full[st], stream_policy);
          ++nk;
          // V runs one tile behind K
          if (nk >= 2 && !load_v(pend_r0, pend_r1)) { ok = false; break; }
          pend_r0 = r0;
          pend_r1 = r1;
        }
      }
      if (ok && nk > nv) load_v(pend_r0, pend_r1);
      // every issued copy has landed before the CTA may exit
      for (int m = max(0, nk - KS); m < nk; ++m) mbar_wait_drain(&bars->k_full[m % KS], (m / KS) & 1, err);
      for (int m = max(0, nv - VS); m < nv; ++m) mbar_wait_drain(&bars->v_full[m % VS], (m / VS) & 1, err);
      for (int m = max(0, nq - 2); m < nq; ++m) mbar_wait_drain(&bars->q_full[m & 1], (m >> 1) & 1, err);
    }
  } else if (warp == 1) {
    // ================================================================ MMA
    if (lane == 0) {
      bool ok = true;
      int n = 0, pi = 0;
      int pv_n = -1, pv_pi = 0;
      bool pv_first = false, pv_last = false;
      auto issue_pv = [&]() {
        const int m = pv_n, ob = pv_pi & 1;
        if (pv_first && !mbar_wait(&bars->o_empty[ob], ((pv_pi >> 1) & 1) ^ 1, err)) return false;
        if (!mbar_wait(&bars->p_full, m & 1, err)) return false;
        if (!mbar_wait(&bars->v_full[m % VS], (m / VS) & 1, err)) return false;
        tc::fence_after_sync();
        const uint32_t v_addr = smem_u32(sV + (m % VS) * C::KV_TILE), p_addr = smem_u32(sP);
#pragma unroll
        for (int kk = 0; kk < BKEY / 16; ++kk)
          tc::mma_bf16_ss(tmem + C::O_COL + ob * 2 * NP,
                          tc::sdesc_sw128(v_addr + (kk / 4) * 2 * C::BOX + (kk % 4) * 2048, C::BOX, 1024),
                          tc::sdesc_sw128(p_addr + (kk / 4) * C::P_BOX + (kk % 4) * 32, 16, 1024), C::IDESC_O,
                          (!pv_first || kk != 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < BKEY / 16; ++kk)   // L += ones . P^T (any 16-key slice of ones is the same)
          tc::mma_bf16_ts(tmem + C::O_COL + ob * 2 * NP + NP, tmem + C::ONES_COL,
                          tc::sdesc_sw128(p_addr + (kk / 4) * C::P_BOX + (kk % 4) * 32, 16, 1024), C::IDESC_S,
                          (!pv_first || kk != 0) ? 1u : 0u);
        tc::mma_commit(&bars->v_empty[m % VS]);
        tc::mma_commit(&bars->p_empty);
        if (pv_last) tc::mma_commit(&bars->o_final[ob]);
        return true;
      };
      PieceWalk w{bars->prefix, U, r_begin, r_end};
      while (ok && w.next()) {
        const int qb = pi & 1;
        for (int t = w.t_lo; t < w.t_hi; ++t, ++n) {
          // S^T of tile n = K_n . Q^T
          if (t == w.t_lo && !mbar_wait(&bars->q_full[qb], (pi >> 1) & 1, err)) { ok = false; break; }
          if (!mbar_wait(&bars->k_full[n % KS], (n / KS) & 1, err)) { ok = false; break; }
          if (n >= 2 && !mbar_wait(&bars->s_free[n & 1], ((n - 2) >> 1) & 1, err)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t k_addr = smem_u32(sK + (n % KS) * C::KV_TILE), q_addr = smem_u32(sQ + qb * C::Q_TILE);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            tc::mma_bf16_ss(tmem + C::S_COL + (n & 1) * NP,
                            tc::sdesc_sw128(k_addr + (kk / 4) * 2 * C::BOX + (kk % 4) * 32, 16, 1024),
                            tc::sdesc_sw128(q_addr + (kk / 4) * C::Q_BOX + (kk % 4) * 32, 16, 1024), C::IDESC_S,
                            kk != 0);
          tc::mma_commit(&bars->k_empty[n % KS]);
          tc::mma_commit(&bars->s_full[n & 1]);
          if (t == w.t_hi - 1) tc::mma_commit(&bars->q_empty[qb]);
          // O^T += V^T P^T of the previous tile, behind the next scores
          if (pv_n >= 0 && !issue_pv()) { ok = false; break; }
          pv_n = n;
          pv_pi = pi;
          pv_first = t == w.t_lo;
          pv_last = t == w.t_hi - 1;
        }
        ++pi;
      }
      if (ok && pv_n >= 0) issue_pv();
      tc::mma_commit(&bars->drain);
      mbar_wait_drain(&bars->drain, 0, err);
    }
  } else if (warp < 6) {
    // ================================================================ softmax
    const int q = warp & 3;                          // TMEM lane quarter
    const int kt = q * 32 + lane;                    // key of the tile (S^T row) / dim (O^T row)
    const int ts = threadIdx.x - 64;                 // 0..127
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const float scale_log2 = 1.4426950408889634f * rsqrtf((float)HD);
    {   // the all-ones A operand of the denominator MMA (bf16 pairs), this warp's lanes
      uint32_t ones[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) ones[i] = 0x3F803F80u;
      asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                   ::"r"(tmem + lane_base + C::ONES_COL), "r"(ones[0]), "r"(ones[1]), "r"(ones[2]), "r"(ones[3]),
                     "r"(ones[4]), "r"(ones[5]), "r"(ones[6]), "r"(ones[7]) : "memory");
      tc::tmem_st_wait();
    }
    int n = 0, pi = 0;
    PieceWalk w{bars->prefix, U, r_begin, r_end};
    while (w.next()) {
      const int b = w.u / p.nkv, ob = pi & 1;
      const int kv_len = bars->lens[b];
      const int tiles_u = bars->prefix[w.u + 1] - bars->prefix[w.u];
      bool broke = false;
      for (int t = w.t_lo; t < w.t_hi; ++t, ++n) {
        const bool valid = t * BKEY + kt < kv_len;
        const bool got = mbar_wait(&bars->s_full[n & 1], (n >> 1) & 1, err);
        if (named_any(1, 128, !got)) { broke = true; break; }
        tc::fence_after_sync();
        float s[NP];
#pragma unroll
        for (int c = 0; c < NP / 16; ++c) {
          uint32_t r[16];
          tc::tmem_ld16(tmem + lane_base + C::S_COL + (n & 1) * NP + c * 16, r);
#pragma unroll
          for (int i = 0; i < 16; ++i) s[c * 16 + i] = __uint_as_float(r[i]);
        }
        tc::tmem_ld_wait();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[n & 1]);
        bool need = false;
#pragma unroll
        for (int h = 0; h < NP; h += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(&bars->m_used[h]);
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            s[h + i] = valid ? s[h + i] * scale_log2 : -INFINITY;
            need |= s[h + i] > mm[i] + kRescaleThreshold;
          }
        }
        need = named_any(1, 128, need);
        if (need) {
          warp_columns<NP, true>(s, bars->red[q]);
          tc::named_sync(1, 128);
          if (ts < NP) {
            const float m_old = bars->m_used[ts];
            const float mt = fmaxf(fmaxf(bars->red[0][ts], bars->red[1][ts]), fmaxf(bars->red[2][ts], bars->red[3][ts]));
            const float m_new = fmaxf(m_old, mt);
            bars->alpha[ts] = m_new == m_old ? 1.f : tc::ex2(m_old - m_new);
            bars->m_used[ts] = m_new;
          }
          tc::named_sync(1, 128);
        }
        // P = 2^(s - m) in registers; the P buffer and O^T are free once the
        // P.V of tile n - 1 has completed
#pragma unroll
        for (int h = 0; h < NP; h += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(&bars->m_used[h]);
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            s[h + i] = tc::ex2(s[h + i] - mm[i]);
          }
        }
        if (n >= 1) mbar_wait(&bars->p_empty, (n - 1) & 1, err);
        if (need && t != w.t_lo) {
          // O^T and L of this piece: column h of each times alpha_h
          {
            tc::fence_after_sync();
#pragma unroll
            for (int c = 0; c < 2 * NP / 16; ++c) {
              uint32_t r[16];
              tc::tmem_ld16(tmem + lane_base + C::O_COL + ob * 2 * NP + c * 16, r);
              tc::tmem_ld_wait();
              const int h0c = (c * 16) % NP;
#pragma unroll
              for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * bars->alpha[h0c + i]);
              tc::tmem_st16(tmem + lane_base + C::O_COL + ob * 2 * NP + c * 16, r);
            }
            tc::tmem_st_wait();
          }
        }
        // P^T as bf16: row h of the B operand holds the tile's 128 keys
        // (K-major, 128-byte swizzle, key halves in two boxes)
        const uint32_t p_row0 = smem_u32(sP) + (kt >> 6) * C::P_BOX + (kt & 7) * 2;
        const int kchunk = (kt & 63) >> 3;
#pragma unroll
        for (int h = 0; h < NP; ++h) {
          const __nv_bfloat16 pb = __float2bfloat16_rn(s[h]);
          st_shared_u16(p_row0 + h * 128 + ((kchunk ^ (h & 7)) << 4), *reinterpret_cast<const uint16_t*>(&pb));
        }
        if (t == tiles_u - 1 && (kv_len % BKEY) != 0) {
          // the unit's last tile: V rows of keys past kv_len -> zeros
          const int st = n % VS;
          const bool landed = mbar_wait(&bars->v_full[st], (n / VS) & 1, err);
          if (!valid && landed) {
            uint8_t* row = sV + st * C::KV_TILE + (kt >> 6) * 2 * C::BOX + (kt & 63) * 128;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              *reinterpret_cast<uint4*>(row + i * 16) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(row + C::BOX + i * 16) = make_uint4(0, 0, 0, 0);
            }
          }
        }
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full);
      }
      if (broke) break;
      // piece end: the running maxima go to the epilogue
      mbar_wait(&bars->ml_empty[ob], ((pi >> 1) & 1) ^ 1, err);
      tc::named_sync(1, 128);
      if (ts < NP) {
        bars->mh[ob][ts] = bars->m_used[ts];
        bars->m_used[ts] = -INFINITY;
      }
      tc::named_sync(1, 128);
      if (ts == 0) mbar_arrive(&bars->ml_full[ob]);
      ++pi;
    }
  } else {
    // ================================================================ epilogue
    const int q = warp & 3;
    const int d = q * 32 + lane;                     // head dimension = O^T row
    const int te = threadIdx.x - 192;                // 0..127
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    constexpr int WS_ROW = HD + kWsPad;
    // units without keys: zero output rows (unit u by CTA u mod grid)
    for (int u = blockIdx.x; u < U; u += gridDim.x) {
      if (bars->prefix[u + 1] != bars->prefix[u]) continue;
      const int b = u / p.nkv, j = u % p.nkv;
      for (int h = 0; h < g; ++h) out[((size_t)b * p.nh + j * g + h) * HD + d] = __float2bfloat16_rn(0.f);
    }
    int pi = 0;
    PieceWalk w{bars->prefix, U, r_begin, r_end};
    while (w.next()) {
      const int b = w.u / p.nkv, j = w.u % p.nkv, ob = pi & 1, ph = (pi >> 1) & 1;
      const int tiles_u = bars->prefix[w.u + 1] - bars->prefix[w.u];
      const bool got = mbar_wait(&bars->o_final[ob], ph, err) && mbar_wait(&bars->ml_full[ob], ph, err);
      if (named_any(2, 128, !got)) break;
      tc::fence_after_sync();
      __nv_bfloat16* orow = out + ((size_t)b * p.nh + j * g) * HD + d;
      float* slot = p.ws + (size_t)(blockIdx.x + w.u) * NP * WS_ROW;
      const bool whole = w.t_lo == 0 && w.t_hi == tiles_u;
      // O^T row d and the denominators (every row of L holds them all), 16 heads at a time:
      // the whole unit is normalised and written; a partial goes to slot (CTA + unit) as
      // o rows, then (m, l) per head
#pragma unroll 1
      for (int c = 0; c < NP / 16; ++c) {
        uint32_t ro[16], rl[16];
        tc::tmem_ld16(tmem + lane_base + C::O_COL + ob * 2 * NP + c * 16, ro);
        tc::tmem_ld16(tmem + lane_base + C::O_COL + ob * 2 * NP + NP + c * 16, rl);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int h = c * 16 + i;
          if (h >= g) continue;
          const float o = __uint_as_float(ro[i]), L = __uint_as_float(rl[i]);
          if (whole) {
            orow[(size_t)h * HD] = __float2bfloat16_rn(L > 0.f ? o / L : 0.f);
          } else {
            slot[h * WS_ROW + d] = o;
            if (d == h) {
              slot[h * WS_ROW + HD] = bars->mh[ob][h];
              slot[h * WS_ROW + HD + 1] = L;
            }
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->o_empty[ob]);
        mbar_arrive(&bars->ml_empty[ob]);
      }
      if (whole) {
        ++pi;
        continue;
      }
      const int c_first = cta_of(bars->prefix[w.u], T, G), c_last = cta_of(bars->prefix[w.u + 1] - 1, T, G);
      const int np = c_last - c_first + 1;
      __threadfence();
      tc::named_sync(2, 128);
      if (te == 0) bars->last = atomicAdd(p.counters + w.u, 1u) == (unsigned)(np - 1);
      tc::named_sync(2, 128);
      const bool last = bars->last != 0;
      ++pi;
      if (!last) continue;
      __threadfence();
      constexpr int SLOT_BYTES = NP * WS_ROW * 4;
      if (w.x >= w.end && np * SLOT_BYTES <= (KS + VS) * C::KV_TILE) {
        // the CTA's last piece: every copy into the K/V ring has been consumed
        // by an MMA that has completed, so the ring takes the np partials, one
        // bulk copy each, and the merge reads them from shared memory
        if (te == 0) {
          asm volatile("fence.proxy.async;" ::: "memory");
          mbar_arrive_expect_tx(&bars->merge_full, np * SLOT_BYTES);
          for (int k = 0; k < np; ++k)
            tc::bulk_load(sK + k * SLOT_BYTES, p.ws + (size_t)(c_first + k + w.u) * NP * WS_ROW, SLOT_BYTES,
                          &bars->merge_full);
        }
        const bool landed = mbar_wait(&bars->merge_full, 0, err);
        if (!named_any(2, 128, !landed)) {
          merge_smem<NP>(reinterpret_cast<const float*>(sK), p, g, b, j, np, te, out);
        } else if (te == 0) {
          mbar_wait_drain(&bars->merge_full, 0, err);   // the copies land before the CTA may exit
        }
      } else {
        merge_unit<NP>(p, g, b, j, c_first + w.u, np, te, out);
      }
      if (te == 0) atomicExch(p.counters + w.u, 0u);  // leave the counter at zero for the next call
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

int sm_count_cached() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 148;
  }
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
    cudaGetLastError();
    v = 148;
  }
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

template <int NP>
cudaError_t launch_np(const DecodeParams& p, cudaStream_t st) {
  constexpr int SMEM = hn_smem_bytes<NP>();
  static_assert(SMEM <= 232448, "227 KB of shared memory per CTA");
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = smem_attr_once(attr_set, reinterpret_cast<const void*>(decode_hn_kernel<NP>), SMEM);
      e != cudaSuccess)
    return e;
  const uint64_t rows = p.block_table ? (uint64_t)p.num_pages * p.nkv * p.page_size : (uint64_t)p.B * p.nkv * p.cap;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16_2d(&tq, p.q, HD, (uint64_t)p.B * p.nh, HD * 2, 64, NP)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tk, p.k_cache, HD, rows, HD * 2, 64, 64)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tv, p.v_cache, HD, rows, HD * 2, 64, 64)) return cudaErrorInvalidValue;
  int grid = sm_count_cached();
  if (grid > kMaxGrid) grid = kMaxGrid;
  return launch_ex(decode_hn_kernel<NP>, dim3((unsigned)grid), dim3(THREADS), SMEM, st, 1u, tq, tk, tv, p, (int)rows);
}

int hn_np(int nh, int nkv) { return (nh / nkv + 15) / 16 * 16; }

}  // namespace

bool decode_hn_ok(int B, int nh, int nkv, int hd, long long cap, bool auto_split) {
  if (hd != HD || !auto_split || nkv <= 0 || nh % nkv) return false;
  const int g = nh / nkv;
  if (g <= 16 || g > 64) return false;
  if ((long long)B * nkv > kMaxUnits) return false;
  return (long long)B * nkv * cap >= kMinKeys;
}

size_t decode_hn_partial_bytes(int B, int nh, int nkv) {
  return (size_t)(kMaxGrid + (size_t)B * nkv) * hn_np(nh, nkv) * (HD + kWsPad) * sizeof(float);
}

cudaError_t launch_decode_hn(const DecodeParams& p, cudaStream_t st) {
  switch (hn_np(p.nh, p.nkv)) {
    case 32: return launch_np<32>(p, st);
    case 48: return launch_np<48>(p, st);
    case 64: return launch_np<64>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gqa
