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
//               bf16 once and store each head to q_out [B, nh, S, hd] or to
//               the cache row [b, j, position]; tiles are 128 tokens x 256
//               fused features, i.e. whole heads, so a rotation pair never
//               leaves the thread that holds it.
//               Output projection: add the residual row in fp32, round once.
//               Both stage their rows in shared memory and write whole
//               128-byte lines (see the staging note below).
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
  // Work items: items below n_full are whole BN-wide tiles; the tiles of a
  // last, partial wave are each cut into two BN/2-wide halves (items n_full
  // and up), so that the last wave keeps twice as many SMs busy for half as
  // long.  Without a partial wave, n_full = num_items = num_tiles.
  int n_full, num_items;
  // K split (ksplit > 1, few-token problems whose tiles would leave most SMs
  // idle): the ksplit CTAs of a cluster each take one tile's k-blocks
  // [rank num_kb / ksplit, (rank + 1) num_kb / ksplit); the ranks above 0
  // leave their partial sums in their shared memory and the leader adds them
  // into its accumulator before the epilogue.  One tile per CTA.
  int ksplit;
};

// Tile of work item i: rows m0.., columns n0.. (width BN or BN/2).
template <int BN, class A>
__device__ __forceinline__ void item_tile(const A& a, int i, int& m0, int& n0, int& width) {
  int t = i, half = 0;
  width = BN;
  if (i >= a.n_full) {
    t = a.n_full + ((i - a.n_full) >> 1);
    half = (i - a.n_full) & 1;
    width = BN / 2;
  }
  m0 = (t / a.num_n) * BM;
  n0 = (t % a.num_n) * BN + half * (BN / 2);
}

struct Bars {
  uint64_t full[MAX_STAGES], empty[MAX_STAGES], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int abort;
  unsigned long long rope_step[64];   // RoPE angle steps in fixed-point turns (rope_turn_step)
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

// Epilogue staging.  Each epilogue warp owns 32 accumulator rows (its TMEM
// lane quarter) and a shared-memory staging area of 32 rows.  A thread first
// writes its own row there (16-byte chunk c of row r at chunk c ^ (r & 7), so
// the 32 rows of a warp spread over all banks); the warp then copies the rows
// out with consecutive lanes on consecutive 16-byte chunks of one row, so
// every store instruction writes whole 128-byte lines of 4 (or 2) rows.
// Row-per-thread stores of 16 bytes would touch 32 lines per instruction,
// and on B200 those partial-line requests slowed the concurrent operand
// stream of the main loop through L2.
__device__ __forceinline__ uint32_t stage_chunk(uint32_t row_base, int r, int c, int mask) {
  return row_base + (uint32_t)((c ^ (r & mask)) * 16);
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a)
               : "memory");
  return v;
}
// 16 bytes global -> shared without registers; src_bytes 0 writes zeros
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// K-split partial sums in shared memory: row r of the tile (BN fp32, i.e.
// BN / 4 chunks of 16 bytes) at r * BN * 4, chunk c at (c & ~7) | ((c ^ r) & 7),
// so that the 32 rows of a warp spread over the banks.
__device__ __forceinline__ uint32_t part_chunk(uint32_t row_base, int r, int c) {
  return row_base + (uint32_t)(((c & ~7) | ((c ^ r) & 7)) * 16);
}
// a rank above 0: its accumulator row (TMEM lane of this thread) -> shared memory
template <int BN>
__device__ __forceinline__ void store_partial(uint32_t tbase, int row, uint32_t part) {
  const uint32_t rb = part + (uint32_t)(row * BN * 4);
#pragma unroll 1
  for (int c = 0; c < BN / 16; ++c) {
    uint32_t v[16];
    __syncwarp();
    tc::tmem_ld16(tbase + c * 16, v);
    tc::tmem_ld_wait();
#pragma unroll
    for (int h = 0; h < 4; ++h)
      tc::st_shared_v4(part_chunk(rb, row, 4 * c + h), v[4 * h], v[4 * h + 1], v[4 * h + 2], v[4 * h + 3]);
  }
}
// the leader: add ranks 1 .. ks-1's rows (read from their shared memory
// across the cluster, a whole row of one rank in flight at a time) into its
// accumulator row
template <int BN>
__device__ __forceinline__ void add_partials(uint32_t tbase, int row, uint32_t part, int ks) {
  constexpr int NCH = BN / 4;   // 16-byte chunks of a row
  const uint32_t rb = part + (uint32_t)(row * BN * 4);
#pragma unroll 1
  for (int q = 1; q < ks; ++q) {
    float4 f[NCH];
#pragma unroll
    for (int c = 0; c < NCH; ++c) f[c] = tc::ld_dsmem_f32x4(tc::mapa_shared(part_chunk(rb, row, c), q));
#pragma unroll
    for (int c = 0; c < BN / 16; ++c) {
      uint32_t v[16];
      __syncwarp();
      tc::tmem_ld16(tbase + c * 16, v);
      tc::tmem_ld_wait();
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        v[4 * h] = __float_as_uint(__uint_as_float(v[4 * h]) + f[4 * c + h].x);
        v[4 * h + 1] = __float_as_uint(__uint_as_float(v[4 * h + 1]) + f[4 * c + h].y);
        v[4 * h + 2] = __float_as_uint(__uint_as_float(v[4 * h + 2]) + f[4 * c + h].z);
        v[4 * h + 3] = __float_as_uint(__uint_as_float(v[4 * h + 3]) + f[4 * c + h].w);
      }
      tc::tmem_st16(tbase + c * 16, v);
    }
    tc::tmem_st_wait();
  }
}

// Epilogue of the QKV projection: RoPE on q/k, head-major scatter.  One
// thread owns token row `row` of the 128 x BN tile at (m0, n0); `tbase` is
// its TMEM lane in the accumulator buffer; `stage` is its warp's staging
// area (32 rows of one head).  A tile holds whole heads, so a rotation pair
// (i, i + hd/2) never leaves the thread that holds it.
template <int HD>
struct QkvEpilogue {
  using Params = QkvParams;
  static constexpr int kStageBytes = 32 * HD * 2;   // per warp: 32 rows of one head
  __device__ static void init(const Params& p, Bars* bars) {
    if (threadIdx.x >= 64 && threadIdx.x < 64 + HD / 2)
      bars->rope_step[threadIdx.x - 64] = rope_turn_step(rope_inv_freq(threadIdx.x - 64, HD, p.theta));
  }
  template <int BN>
  __device__ static void prefetch(const TcArgs<Params>&, int, int, int, uint32_t) {}
  template <int BN>
  __device__ static void tile(const TcArgs<Params>& a, const Bars* bars, uint32_t tbase, int m0, int n0, int row,
                              uint32_t stage) {
    constexpr int HALF = HD / 2, CHUNKS = HALF / 16, HEADS = BN / HD;
    constexpr int ROWB = HD * 2, RCH = ROWB / 16;          // bytes and 16-byte chunks of a head row
    constexpr int MASK = RCH < 8 ? RCH - 1 : 7;
    constexpr int LPR = RCH, RPI = 32 / LPR;               // copy-out: lanes per row, rows per instruction
    static_assert(BN % HD == 0, "tiles hold whole heads");
    const Params& p = a.p;
    int* err = p.err;
    const int lane = threadIdx.x % 32;
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
    const uint32_t my_row = stage + lane * ROWB;
    const int cc = lane % LPR, rsub = lane / LPR;
#pragma unroll 1
    for (int hh = 0; hh < HEADS; ++hh) {
      const int hb = hb0 + hh;
      if (hb >= a.n_heads_total) break;  // ragged N tail: uniform over the CTA
      const bool is_q = hb < p.nh, is_k = !is_q && hb < p.nh + p.nkv;
      __nv_bfloat16* dst = nullptr;
      if (valid) {
        if (is_q) {
          dst = static_cast<__nv_bfloat16*>(p.q_out) + (((size_t)b * p.nh + hb) * p.S + s) * HD;
        } else if (pos_ok) {
          const int j = is_k ? hb - p.nh : hb - p.nh - p.nkv;
          dst = static_cast<__nv_bfloat16*>(is_k ? p.k_cache : p.v_cache) +
                (((size_t)b * p.nkv + j) * p.cap + pos) * HD;
        } else {
          raise_error(err, GQA_DEVERR_POSITION_RANGE);
        }
      }
#pragma unroll 1
      for (int c = 0; c < CHUNKS; ++c) {
        uint32_t lo[16], hi[16];
        __syncwarp();  // the .sync.aligned TMEM load needs the whole warp converged
        tc::tmem_ld16(tbase + hh * HD + c * 16, lo);
        tc::tmem_ld16(tbase + hh * HD + HALF + c * 16, hi);
        uint32_t olo[8], ohi[8];
        if (is_q || is_k) {
          float cs[16], sn[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) rope_cos_sin_fx(pos, bars->rope_step[c * 16 + k], &cs[k], &sn[k]);
          tc::tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; k += 2) {
            const float x0 = __uint_as_float(lo[k]), y0 = __uint_as_float(hi[k]);
            const float x1 = __uint_as_float(lo[k + 1]), y1 = __uint_as_float(hi[k + 1]);
            olo[k / 2] = pack_bf16x2(x0 * cs[k] - y0 * sn[k], x1 * cs[k + 1] - y1 * sn[k + 1]);
            ohi[k / 2] = pack_bf16x2(y0 * cs[k] + x0 * sn[k], y1 * cs[k + 1] + x1 * sn[k + 1]);
          }
        } else {
          tc::tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; k += 2) {
            olo[k / 2] = pack_bf16x2(__uint_as_float(lo[k]), __uint_as_float(lo[k + 1]));
            ohi[k / 2] = pack_bf16x2(__uint_as_float(hi[k]), __uint_as_float(hi[k + 1]));
          }
        }
        // features c*16.. and HALF + c*16.. of the head row: chunks 2c, 2c+1 and RCH/2 + 2c, +1
        tc::st_shared_v4(stage_chunk(my_row, lane, 2 * c, MASK), olo[0], olo[1], olo[2], olo[3]);
        tc::st_shared_v4(stage_chunk(my_row, lane, 2 * c + 1, MASK), olo[4], olo[5], olo[6], olo[7]);
        tc::st_shared_v4(stage_chunk(my_row, lane, RCH / 2 + 2 * c, MASK), ohi[0], ohi[1], ohi[2], ohi[3]);
        tc::st_shared_v4(stage_chunk(my_row, lane, RCH / 2 + 2 * c + 1, MASK), ohi[4], ohi[5], ohi[6], ohi[7]);
      }
      __syncwarp();
      // copy-out: instruction i writes rows i*RPI .. i*RPI + RPI-1, LPR lanes per row
#pragma unroll
      for (int i = 0; i < 32 / RPI; ++i) {
        const int rr = i * RPI + rsub;
        const unsigned long long d = __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dst), rr);
        const uint4 v = ld_shared_v4(stage_chunk(stage + rr * ROWB, rr, cc, MASK));
        if (d) tc::st_global_v4(reinterpret_cast<uint8_t*>(d) + cc * 16, v.x, v.y, v.z, v.w);
      }
      __syncwarp();  // the staging rows are rewritten by the next head
    }
  }
};

// Epilogue of the output projection: out = acc + residual, rounded once.
// The tile's columns go in groups of 64 (one 128-byte staging row per
// thread).  The residual of each group is fetched into the staging area with
// coalesced cp.async copies, double-buffered: group 0 is requested before the
// accumulator is ready, group g + 1 while group g is added and stored.  The
// thread owning a row adds its accumulator columns to the staged residual in
// place, then the warp copies the rows out as whole lines.  Columns go in
// 8-wide vectors; a vector past N (N % 8 == 0) is neither read nor written,
// so a ragged N tail needs no masking inside a vector.  out may be the
// residual buffer: a tile's residual is read before its output is written,
// and no other CTA touches the tile.
struct ResidualEpilogue {
  using Params = OprojParams;
  static constexpr int G = 64;                         // columns per group
  static constexpr int kBufBytes = 32 * G * 2;         // one group of 32 rows
  static constexpr int kStageBytes = 2 * kBufBytes;    // double-buffered
  __device__ static void init(const Params&, Bars*) {}
  // cp.async of the residual's group g (rows m0 + 32w .. +31) into buffer g & 1
  template <int BN>
  __device__ static void fetch(const Params& p, int T, int m0w, int n0, int g, uint32_t stage) {
    const int lane = threadIdx.x % 32, cc = lane % 8, rsub = lane / 8;
    const uint32_t buf = stage + (g & 1) * kBufBytes;
    const __nv_bfloat16* res = static_cast<const __nv_bfloat16*>(p.residual);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int rr = i * 4 + rsub, t = m0w + rr, n = n0 + g * G + cc * 8;
      const bool in = t < T && n < p.N;
      cp_async_16(stage_chunk(buf + rr * 128, rr, cc, 7), in ? res + (size_t)t * p.N + n : res, in ? 16 : 0);
    }
    cp_async_commit();
  }
  template <int BN>
  __device__ static void prefetch(const TcArgs<Params>& a, int m0, int n0, int q4, uint32_t stage) {
    if (a.p.residual) fetch<BN>(a.p, a.T, m0 + 32 * q4, n0, 0, stage);
  }
  template <int BN>
  __device__ static void tile(const TcArgs<Params>& a, const Bars*, uint32_t tbase, int m0, int n0, int row,
                              uint32_t stage) {
    constexpr int NG = BN / G;
    const Params& p = a.p;
    const bool has_res = p.residual != nullptr;
    const int lane = threadIdx.x % 32, cc = lane % 8, rsub = lane / 8;
    const int m0w = m0 + (row - lane);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
#pragma unroll 1
    for (int g = 0; g < NG; ++g) {
      if (n0 + g * G >= p.N) break;  // uniform over the CTA
      const uint32_t buf = stage + (g & 1) * kBufBytes;
      if (has_res) {
        if (g + 1 < NG && n0 + (g + 1) * G < p.N) {
          fetch<BN>(p, a.T, m0w, n0, g + 1, stage);
          cp_async_wait<1>();
        } else {
          cp_async_wait<0>();
        }
      }
      __syncwarp();
      const uint32_t my_row = buf + lane * 128;
#pragma unroll
      for (int c = 0; c < G / 16; ++c) {
        uint32_t v[16];
        __syncwarp();
        tc::tmem_ld16(tbase + g * G + c * 16, v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t addr = stage_chunk(my_row, lane, 2 * c + h, 7);
          float f[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(v[8 * h + k]);
          if (has_res) {
            const uint4 r = ld_shared_v4(addr);
            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&rw[k]);
              f[2 * k] += __low2float(b2);
              f[2 * k + 1] += __high2float(b2);
            }
          }
          tc::st_shared_v4(addr, pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                           pack_bf16x2(f[6], f[7]));
        }
      }
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = i * 4 + rsub, t = m0w + rr, n = n0 + g * G + cc * 8;
        const uint4 v = ld_shared_v4(stage_chunk(buf + rr * 128, rr, cc, 7));
        if (t < a.T && n < p.N) tc::st_global_v4(out + (size_t)t * p.N + n, v.x, v.y, v.z, v.w);
      }
      __syncwarp();  // this buffer takes group g + 2
    }
  }
};

template <class Epi, class Cfg>
__global__ void __launch_bounds__(THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
               const __grid_constant__ CUtensorMap tmw_half, TcArgs<typename Epi::Params> a) {
  constexpr int BN = Cfg::BN, STAGES = Cfg::STAGES, A_BYTES = Cfg::A_BYTES, STAGE_BYTES = Cfg::STAGE_BYTES;
  constexpr int TMEM_COLS = Cfg::TMEM_COLS;
  constexpr uint32_t IDESC = Cfg::IDESC;
  constexpr uint32_t IDESC_HALF = tc::idesc_bf16(BM, BN / 2, false, false);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int* err = a.p.err;
  pdl_launch_dependents();

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
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmx);
    tc::prefetch_tmap(&tmw);
    if (a.num_items > a.n_full) tc::prefetch_tmap(&tmw_half);
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, TMEM_COLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  pdl_wait();   // the inputs may come from the kernel before this one
  // K split: rank within the cluster, its k-blocks, and one tile per CTA
  const int ks = a.ksplit, rank = ks > 1 ? (int)(blockIdx.x % ks) : 0;
  const int item0 = ks > 1 ? (int)(blockIdx.x / ks) : (int)blockIdx.x;
  const int item_step = ks > 1 ? a.num_items : (int)gridDim.x;
  const int kb0 = rank * a.num_kb / ks, kb1 = (rank + 1) * a.num_kb / ks;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int item = item0; ok && item < a.num_items; item += item_step) {
        int m0, n0, width;
        item_tile<BN>(a, item, m0, n0, width);
        const CUtensorMap* wmap = width == BN ? &tmw : &tmw_half;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&bars->empty[stage], phase ^ 1, err)) { ok = false; break; }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&bars->full[stage], A_BYTES + width * BK * 2);
          tc::tma_load_2d(sa, &tmx, kb * BK, m0, &bars->full[stage]);
          tc::tma_load_2d(sa + A_BYTES, wmap, kb * BK, n0, &bars->full[stage]);
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
      for (int item = item0; ok && item < a.num_items; item += item_step, ++it) {
        const int buf = it & 1;
        const uint32_t idesc = item < a.n_full ? IDESC : IDESC_HALF;
        if (!mbar_wait(&bars->acc_empty[buf], ((it >> 1) & 1) ^ 1, err)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t d = tmem + buf * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&bars->full[stage], phase, err)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            tc::mma_bf16_ss(d, tc::sdesc_sw128(sa + k * 32, 16, 1024), tc::sdesc_sw128(sb + k * 32, 16, 1024),
                            idesc, kb > kb0 || k != 0);
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
    const uint32_t stage = smem_u32(smem + STAGES * STAGE_BYTES + 1024) + q4 * Epi::kStageBytes;
    // the epilogue's table (RoPE angle steps), made while the first loads fly
    Epi::init(a.p, bars);
    tc::named_sync(1, 128);
    int it = 0;
    for (int item = item0; item < a.num_items; item += item_step, ++it) {
      const int buf = it & 1;
      int m0, n0, width;
      item_tile<BN>(a, item, m0, n0, width);
      if (rank == 0) Epi::template prefetch<BN>(a, m0, n0, q4, stage);
      const bool got = mbar_wait(&bars->acc_full[buf], (it >> 1) & 1, err);
      if (!__all_sync(0xffffffffu, got)) break;
      tc::fence_after_sync();
      const uint32_t tbase = tmem + ((uint32_t)(q4 * 32) << 16) + buf * BN;
      if (ks > 1) {
        // K split: the leader's epilogue runs once every rank's sums are in
        if constexpr (BN <= 128) {
          if (rank > 0) store_partial<BN>(tbase, row, smem_u32(smem));
        }
        break;
      }
      if constexpr (BN == 256) {
        if (width == BN) Epi::template tile<BN>(a, bars, tbase, m0, n0, row, stage);
        else Epi::template tile<BN / 2>(a, bars, tbase, m0, n0, row, stage);
      } else {
        Epi::template tile<BN>(a, bars, tbase, m0, n0, row, stage);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
    }
    cp_async_wait<0>();  // no staging copy outlives the CTA
  }

  tc::fence_before_sync();
  __syncthreads();
  if constexpr (BN <= 128) {
    if (ks > 1) {
      // every rank's partial sums are in its shared memory
      tc::cluster_sync();
      if (rank == 0 && warp >= 2 && !*reinterpret_cast<volatile int*>(&bars->abort)) {
        tc::fence_after_sync();
        const int q4 = warp & 3, row = q4 * 32 + lane;
        const uint32_t stage = smem_u32(smem + STAGES * STAGE_BYTES + 1024) + q4 * Epi::kStageBytes;
        const uint32_t tbase = tmem + ((uint32_t)(q4 * 32) << 16);
        int m0, n0, width;
        item_tile<BN>(a, item0, m0, n0, width);
        add_partials<BN>(tbase, row, smem_u32(smem), ks);
        Epi::template tile<BN>(a, bars, tbase, m0, n0, row, stage);
        cp_async_wait<0>();
      }
      // no rank leaves while the leader may still read its shared memory
      tc::cluster_sync();
      tc::fence_before_sync();
      __syncthreads();
    }
  }
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <class Epi, class Cfg>
cudaError_t launch_cfg(const typename Epi::Params& p, const void* x, const void* w, int T, int K, int N,
                       int n_heads_total, int num_sms, cudaStream_t st, int ksplit = 1) {
  constexpr int SMEM = Cfg::SMEM_BYTES + 4 * Epi::kStageBytes;
  static_assert(SMEM <= 232448, "227 KB of shared memory per CTA");
  static std::atomic<bool> attr_set[64];
  if (cudaError_t e = smem_attr_once(attr_set, reinterpret_cast<const void*>(gemm_tc_kernel<Epi, Cfg>), SMEM);
      e != cudaSuccess)
    return e;
  TcArgs<typename Epi::Params> a;
  a.p = p;
  a.T = T;
  a.n_heads_total = n_heads_total;
  a.num_n = (N + Cfg::BN - 1) / Cfg::BN;
  a.num_tiles = ((T + BM - 1) / BM) * a.num_n;
  a.num_kb = (K + BK - 1) / BK;
  // a partial last wave of wide tiles goes as twice as many half-width tiles
  // when they still fit in one wave
  a.ksplit = ksplit;
  const int rem = num_sms > 0 ? a.num_tiles % num_sms : 0;
  if (Cfg::BN == 256 && ksplit == 1 && a.num_tiles > num_sms && rem > 0 && 2 * rem <= num_sms) {
    a.n_full = a.num_tiles - rem;
    a.num_items = a.num_tiles + rem;
  } else {
    a.n_full = a.num_items = a.num_tiles;
  }
  CUtensorMap tx, tw, tw_half;
  if (!make_tmap_bf16_2d(&tx, x, K, T, (uint64_t)K * 2, BK, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tw, w, K, N, (uint64_t)K * 2, BK, Cfg::BN)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tw_half, w, K, N, (uint64_t)K * 2, BK, Cfg::BN / 2)) return cudaErrorInvalidValue;
  // K split: one tile per CTA, the ksplit CTAs of a tile in one cluster
  const int grid = ksplit > 1 ? a.num_tiles * ksplit : (a.num_items < num_sms ? a.num_items : num_sms);
  return launch_ex(gemm_tc_kernel<Epi, Cfg>, dim3((unsigned)grid), dim3(THREADS), SMEM, st, (unsigned)ksplit,
                   tx, tw, tw_half, a);
}

// K split for problems whose narrow tiles fill less than half of the SMs:
// two CTAs per tile, each with at least 4 k-blocks.  Measured on B200 (128
// tokens, hidden 2048): 3 or 4 ranks were no faster than 2 for the QKV
// projection and slower for the output projection (the leader reads more
// partials), and 48 clusters of 3 CTAs of ~210 KB did not all fit at once.
inline int ksplit_for(long long tiles, int num_kb, int num_sms) {
  if (tiles <= 0 || 2 * tiles > num_sms || num_kb < 8) return 1;
  return 2;
}

// Wide tiles unless they would leave more than half of the SMs idle; then
// the narrowest tile that still holds whole heads (`min_bn`).
template <class Epi, int MIN_BN>
cudaError_t launch_gemm(const typename Epi::Params& p, const void* x, const void* w, int T, int K, int N,
                        int n_heads_total, int num_sms, cudaStream_t st) {
  const long long wide_tiles = (long long)((T + BM - 1) / BM) * ((N + 255) / 256);
  if (2 * wide_tiles >= num_sms) return launch_cfg<Epi, GemmCfg<256, 4>>(p, x, w, T, K, N, n_heads_total, num_sms, st);
  constexpr int NBN = MIN_BN <= 64 ? 64 : 128;
  const long long tiles = (long long)((T + BM - 1) / BM) * ((N + NBN - 1) / NBN);
  const int ks = ksplit_for(tiles, (K + BK - 1) / BK, num_sms);
  if constexpr (MIN_BN <= 64)
    return launch_cfg<Epi, GemmCfg<64, 8>>(p, x, w, T, K, N, n_heads_total, num_sms, st, ks);
  else
    return launch_cfg<Epi, GemmCfg<128, 6>>(p, x, w, T, K, N, n_heads_total, num_sms, st, ks);
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
