/*
 * gqa.h - C ABI of the B200 (sm_100a) fused-QKV + grouped-query attention
 * library (libgqa_b200.so).
 *
 * Three calls form the path of one Llama-style attention layer:
 *
 *   qkv_rope_project   hidden states -> one fused W_qkv GEMM -> RoPE on q/k ->
 *                      q written head-major, k/v written into the KV cache
 *   gqa_attn_prefill   exact (online-softmax) attention of S new queries per
 *                      sequence over the cache, causal or not
 *   gqa_attn_decode    one new query per sequence over a ragged-length cache,
 *                      split along the keys, partials merged by log-sum-exp
 *
 * Grouped-query attention: n_heads query heads share n_kv_heads key/value
 * heads, g = n_heads / n_kv_heads consecutive query heads per KV head (query
 * head h reads KV head h / g).  MHA is n_kv_heads == n_heads, MQA is
 * n_kv_heads == 1.
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller; the library
 *   never allocates, frees, synchronises or prints.  Every call is
 *   asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the
 *   legacy default stream) and may be captured in a CUDA graph.
 * - Kernels are launched with programmatic stream serialization: a kernel of
 *   the library may start while the kernel before it on `stream` is still
 *   running, and waits for it (griddepcontrol.wait) before its first access
 *   to global memory, so stream order holds for every buffer.  Each library
 *   kernel also lets the next kernel on the stream launch early; a kernel of
 *   the caller's that follows a library call and is itself launched with the
 *   programmatic-serialization attribute must call
 *   cudaGridDependencySynchronize() before it reads the call's outputs
 *   (kernels launched without that attribute wait for completion as usual).
 * - Tensors are dense, row-major ("C order") with the shapes given below, and
 *   every tensor pointer must be 16-byte aligned (int32 arrays: 4-byte).
 * - dtype: GQA_F32 (float32 everywhere, FFMA arithmetic, no TF32) or
 *   GQA_BF16 (bfloat16 storage, float32 accumulation; P is rounded to bf16
 *   before the P.V product, outputs are rounded once to nearest-even).
 * - Return value: GQA_OK (0) or a negative GQA_ERR_* code.  Arguments are
 *   validated on the host only; device data (positions, kv_lens) is never
 *   read by the host.  Device-side range problems (a position outside
 *   [0, cache_cap), a kv_len above cache_cap) are clamped or skipped as
 *   documented per call and recorded in a device error word that
 *   gqa_device_error() reads.
 * - head_dim must be 32, 64 or 128; B == 0 or S == 0 is a valid no-op.
 * - Size limits (GQA_ERR_UNSUPPORTED_SHAPE beyond them): every tensor below
 *   2^40 elements; B and n_heads (prefill) or n_kv_heads (decode) at most
 *   65535; fewer than 2^31 cache rows (B * n_kv_heads * cache_cap, or
 *   num_pages * n_kv_heads * page_size for a paged cache), query rows
 *   (B * n_heads * S) and tokens (B * S).
 * - Runs only on compute capability 10.0 devices (B200, sm_100a).
 */
#ifndef GQA_B200_H
#define GQA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum gqa_dtype { GQA_F32 = 0, GQA_BF16 = 1 };

enum gqa_status {
  GQA_OK = 0,
  GQA_ERR_INVALID_ARG = -1,        /* null pointer, negative size, nh % nkv != 0, ... */
  GQA_ERR_MISALIGNED = -2,         /* a tensor pointer is not 16-byte aligned */
  GQA_ERR_UNSUPPORTED_DTYPE = -3,  /* dtype is neither GQA_F32 nor GQA_BF16 */
  GQA_ERR_UNSUPPORTED_ARCH = -4,   /* current device is not compute capability 10.0 */
  GQA_ERR_WORKSPACE_TOO_SMALL = -5,/* decode workspace smaller than the size query */
  GQA_ERR_LAUNCH_FAILED = -6,      /* a kernel launch returned a CUDA error */
  GQA_ERR_UNSUPPORTED_SHAPE = -7,  /* head_dim not in {32, 64, 128} or a size too large */
  GQA_ERR_NO_DEVICE = -8           /* no CUDA device is current */
};

/* Device error word bits (gqa_device_error). */
enum gqa_device_error_bits {
  GQA_DEVERR_POSITION_RANGE = 1,   /* a position outside [0, cache_cap): K/V row not written */
  GQA_DEVERR_KVLEN_RANGE = 2,      /* a kv_len above cache_cap (clamped) or below 0 (taken as 0) */
  GQA_DEVERR_WAIT_TIMEOUT = 4,     /* a pipeline wait gave up after its time limit */
  GQA_DEVERR_PAGE_RANGE = 8,       /* a block-table entry outside [0, num_pages): read as zeros */
  GQA_DEVERR_SEQLEN_RANGE = 16     /* packed offsets decreasing or past the tensors (clamped), or a
                                      query run longer than max_seqlen_q (rows past it not written) */
};

/*
 * qkv_rope_project - steps a1..a3 of the path.
 *
 * Source: "Optimize LlamaAttention by fusing QKV projections"
 * (huggingface/transformers pull request #40092), LlamaAttention.forward:
 * one qkv_proj linear layer whose output is sliced into query features
 * [0, nh*hd), key features [nh*hd, (nh+nkv)*hd) and value features
 * [(nh+nkv)*hd, (nh+2nkv)*hd); head j of a block owns features j*hd..j*hd+hd-1.
 * RoPE (rotate_half pairing: feature i with i + hd/2, inv_freq_i =
 * theta^(-2i/hd), angle = position * inv_freq_i) is applied to q and k only
 * (the fused-QKV toy model of the custom-op overhead gist also applies its
 * position step to q and k after the split).
 *
 *   x          [B, S, hidden]                      dtype
 *   w_qkv      [(n_heads + 2 n_kv_heads) * head_dim, hidden]  dtype
 *              (nn.Linear storage: y = x w^T, no bias)
 *   positions  [B, S] int32: absolute position of each token; it sets the
 *              rotation angle and the cache slot of its K/V rows
 *   q_out      [B, n_heads, S, head_dim] dtype (written, head-major)
 *   k_cache,
 *   v_cache    [B, n_kv_heads, cache_cap, head_dim] dtype; row positions[b,s]
 *              of every KV head of sequence b is overwritten, all other rows
 *              are left untouched.  A position outside [0, cache_cap) writes
 *              no K/V row and sets GQA_DEVERR_POSITION_RANGE (q is still
 *              written, rotated by that position).  Two tokens of one
 *              sequence with the same position write the same row; which
 *              one lands is unspecified.
 *
 * The math is float32 (fp32 accumulation of bf16 products for GQA_BF16), with
 * one final rounding of q/k/v to dtype.
 */
int qkv_rope_project(const void* x, const void* w_qkv, const int32_t* positions,
                     int B, int S, int hidden, int n_heads, int n_kv_heads, int head_dim,
                     float rope_theta, void* q_out, void* k_cache, void* v_cache,
                     int cache_cap, int dtype, void* stream);

/*
 * gqa_attn_prefill - step a4: exact attention of S queries per sequence.
 *
 * Source: "FlashAttention-3" (together.ai summary), section
 * "FlashAttention方式のおさらい": tiled attention with softmax rescaling gives
 * the exact softmax(Q K^T / sqrt(hd)) V without writing the score matrix;
 * "MHA -> GQA" blog, section 3.2: g query heads share one KV head.
 *
 *   q            [B, n_heads, S, head_dim] dtype (as written by qkv_rope_project)
 *   k_cache,
 *   v_cache      [B, n_kv_heads, cache_cap, head_dim] dtype
 *   q_positions  [B, S] int32 or NULL.  NULL means kv_lens[b] - S + s
 *                (the S queries are the last S cached tokens).
 *   kv_lens      [B] int32: keys 0..kv_lens[b]-1 of sequence b are valid;
 *                values above cache_cap are clamped (GQA_DEVERR_KVLEN_RANGE).
 *   causal       nonzero: key t is visible to a query at position p iff t <= p
 *   out          [B, S, n_heads, head_dim] dtype (token-major, ready for an
 *                output projection).  A query with no visible key gets zeros.
 *
 * Scale 1/sqrt(head_dim).  Cache rows at or beyond kv_len are never read
 * into the result (they may hold anything, NaN included).
 */
int gqa_attn_prefill(const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* q_positions, const int32_t* kv_lens,
                     int B, int S, int n_heads, int n_kv_heads, int head_dim,
                     int cache_cap, int causal, void* out, int dtype, void* stream);

/*
 * gqa_attn_prefill_varlen - gqa_attn_prefill over packed variable-length
 * sequences.
 *
 * Source: "FlashAttention-3" (together.ai summary), section "残る最適化と今後の
 * 統合": the paper adds variable-length sequences.  Read as the packed
 * layout of the FlashAttention library: the sequences of a batch are
 * concatenated along the token axis and delimited by cumulative offsets, so
 * no padding is stored, read or computed.  Sequence b owns query rows
 * [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key/value rows
 * [cu_seqlens_k[b], cu_seqlens_k[b+1]) and attends to its own keys only.
 * With Sq queries over Sk keys, query s sits at position Sk - Sq + s
 * (bottom-right, as the padded call's default), and when causal sees the
 * keys at positions <= its own; a query that sees no key gets a zero row.
 *
 *   q             [total_q, n_heads, head_dim] bf16 (token-major, packed)
 *   k, v          [total_k, n_kv_heads, head_dim] bf16
 *   cu_seqlens_q,
 *   cu_seqlens_k  [B + 1] int32, non-decreasing, from 0 to total_q / total_k.
 *                 Offsets outside the tensors, or decreasing, are clamped
 *                 and raise GQA_DEVERR_SEQLEN_RANGE
 *   max_seqlen_q  the longest query run (sizes the grid); a longer run raises
 *                 GQA_DEVERR_SEQLEN_RANGE and its rows past the grid are not
 *                 written
 *   out           [total_q, n_heads, head_dim] bf16
 *
 * bf16 with head_dim 64 or 128 only.  total_q == 0, B == 0 or
 * max_seqlen_q == 0 is a no-op; total_k may be 0 (zero rows).  Statuses as
 * gqa_attn_prefill; asynchronous on `stream`.
 */
int gqa_attn_prefill_varlen(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                            const int32_t* cu_seqlens_k, int B, int total_q, int total_k, int max_seqlen_q,
                            int n_heads, int n_kv_heads, int head_dim, int causal, void* out, int dtype,
                            void* stream);

/*
 * gqa_attn_decode_workspace_size - bytes of device workspace gqa_attn_decode
 * needs for these sizes: a block of split counters (one 32-bit word per
 * sequence, KV head and group of up to 16 query heads, rounded up to 256
 * bytes) followed by float32 partial results (a running max, a sum and an
 * unnormalised output row per sequence, query head and key split).  When the
 * split is left to the library and the problem may take the decode that cuts
 * the sequences' keys into equal ranges per SM (head_dim 128, 17..64 query
 * heads per KV head, at least 2^18 cached key rows, at most 512 sequence x
 * KV head pairs), the partials take at most (160 + B * n_kv_heads) slots of
 * n_heads / n_kv_heads (rounded up to 16) rows of head_dim + 4 floats, and
 * the size covers the larger of the two layouts.
 * kv_split: keys per split, 0 = the library's choice, else a multiple of 64.
 * Returns 0 for invalid arguments.
 */
size_t gqa_attn_decode_workspace_size(int B, int n_heads, int n_kv_heads, int head_dim,
                                      int cache_cap, int kv_split);

/*
 * gqa_attn_decode - steps a5..a6: one new query per sequence.
 *
 * Source: "MHA -> GQA" blog, sections 3.1-3.2: decode attention is a batched
 * matrix-vector product over ragged lengths and stays memory-bound; the g
 * query heads that share a KV head are processed together so that every
 * K/V byte read serves g heads (arithmetic intensity ~g).  The keys of a
 * sequence are split into chunks of kv_split; each chunk produces a partial
 * (max m, sum l, unnormalised o) per head and the partials are merged with a
 * log-sum-exp combine, which is exact.  On the tensor-core path (bf16,
 * head_dim 64/128) the last chunk of a (sequence, KV head) to finish does the
 * merge, found through a counter in the workspace (or, for the library's own
 * split of small caches, inside a thread-block cluster); a sequence with a
 * single chunk is written directly.  Large problems with 17..64 query heads
 * per KV head at head_dim 128 whose cache is paged or longer than 8 x 2048
 * keys cut the concatenated 128-key tiles of all sequences into one equal
 * range per SM instead; its pieces merge the same way.
 *
 *   q          [B, n_heads, head_dim] dtype (the new token, already rotated)
 *   k_cache,
 *   v_cache    [B, n_kv_heads, cache_cap, head_dim] dtype
 *   kv_lens    [B] int32: valid keys including the new token; clamped to
 *              [0, cache_cap] (GQA_DEVERR_KVLEN_RANGE); 0 gives a zero row
 *   kv_split   keys per split: 0 = automatic, else a positive multiple of 64
 *              giving at most 512 splits of cache_cap
 *   out        [B, n_heads, head_dim] dtype
 *   workspace  device scratch of at least gqa_attn_decode_workspace_size()
 *              bytes, 16-byte aligned, ZERO-FILLED BEFORE ITS FIRST USE
 *              (e.g. cudaMemset once after allocating it).  Every call leaves
 *              the counter block at zero again, so a workspace can be reused
 *              by any later call; calls that may run at the same time on the
 *              GPU need workspaces of their own.
 */
int gqa_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* kv_lens, int B, int n_heads, int n_kv_heads, int head_dim,
                    int cache_cap, int kv_split, void* out, void* workspace,
                    size_t workspace_bytes, int dtype, void* stream);

/*
 * gqa_attn_decode_noalloc - gqa_attn_decode without a workspace argument.
 *
 * The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory where they run decode: a serving loop whose
 * device memory is all pre-reserved by another allocator, a plugin that its
 * host framework hands only the op's tensors (no allocator interface), or a
 * latency-critical path on which an allocation, which may synchronise the
 * device, is not allowed.  The caller still passes every input and output;
 * arguments, layouts, results and argument checks are those of
 * gqa_attn_decode (both run the same validation), except that a problem too
 * large for the static scratch returns GQA_ERR_WORKSPACE_TOO_SMALL.
 *
 * The split counters and partials live in a fixed 64 MiB array of static
 * device memory inside the library, which every GPU that loads the library
 * holds until the process exits.  A problem whose workspace
 * (gqa_attn_decode_workspace_size) exceeds 64 MiB is rejected with
 * GQA_ERR_WORKSPACE_TOO_SMALL; a larger kv_split needs fewer partials.
 * The first call on each device looks up the array's device address, with
 * that device current (a host-side runtime query; make that first call
 * before any stream capture).  Every call then clears the counter block at
 * the front of the array with cudaMemsetAsync on `stream`, before its decode
 * kernel on the same stream, because the array keeps whatever the previous
 * call left there.  All calls share the array: calls that overlap on the
 * GPU (e.g. on two streams) race, so order them on one stream or with
 * events.  It allocates nothing.
 */
int gqa_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* kv_lens, int B, int n_heads, int n_kv_heads, int head_dim,
                            int cache_cap, int kv_split, void* out, int dtype, void* stream);

/*
 * gqa_o_proj_residual - the attention layer's output projection with the
 * residual add (the step after a4 / a5).
 *
 * Source: the "custom op overhead" gist (youkaichao), toy model:
 * LlamaAttention.forward ends in output = self.output_projection(attn_output),
 * a linear layer from the n_heads * head_dim concatenated head outputs back to
 * the hidden size, and LlamaDecoderLayer adds that output to the residual
 * stream.  (The toy's linear layers carry a bias; the layer here has none, as
 * W_qkv has none.)
 *
 *   attn      [T, n_heads, head_dim] dtype: per token the heads in order,
 *             i.e. [T, n_heads * head_dim] (gqa_attn_prefill's out
 *             [B, S, n_heads, head_dim] with T = B * S, or gqa_attn_decode's
 *             out [B, n_heads, head_dim] with T = B)
 *   w_o       [hidden, n_heads * head_dim] dtype (nn.Linear storage: y = x w^T)
 *   residual  [T, hidden] dtype, or NULL for none
 *   out       [T, hidden] dtype: out = attn . w_o^T + residual, accumulated in
 *             float32 (the residual added in float32) and rounded once.  out
 *             may be the residual buffer itself (an in-place update of the
 *             residual stream); it must not overlap attn or w_o.
 *
 * bf16 with hidden % 8 == 0 runs on the tensor cores (tcgen05): 128-token
 * tiles, or for T <= 64 tiles whose rows are 128 rows of w_o with the
 * reduction split over a thread-block cluster.  float32 (FFMA, no TF32) and
 * other bf16 widths run a SIMT kernel.  T == 0 is a no-op.
 * Errors: GQA_ERR_INVALID_ARG (null pointers, non-positive sizes, out
 * overlapping attn or w_o, or partly overlapping the residual),
 * GQA_ERR_UNSUPPORTED_SHAPE (head_dim, sizes), GQA_ERR_MISALIGNED,
 * GQA_ERR_UNSUPPORTED_DTYPE and the device/launch statuses.  Asynchronous on
 * `stream`; allocates nothing.
 */
int gqa_o_proj_residual(const void* attn, const void* w_o, const void* residual, int T, int n_heads,
                        int head_dim, int hidden, void* out, int dtype, void* stream);

/*
 * gqa_meanpool_kv_heads - MHA -> GQA weight transform ("MHA -> GQA: 提升 LLM
 * 推理效率", section 4.3: the new KV projection of each group of heads is
 * initialised by mean pooling the group's projections).
 *
 * From a fused MHA weight it writes the fused GQA weight with n_kv_heads KV
 * heads: query rows copied; key (value) row j*head_dim + d of the result is
 * the mean of rows (j*g + i)*head_dim + d, i < g = n_heads / n_kv_heads, of
 * the MHA key (value) block.  The groups are the consecutive heads that the
 * attention calls map onto one KV head (h -> h / g).  Sums in fp32, one
 * rounding to the dtype.
 *
 *   w_qkv_mha  [3 * n_heads * head_dim, hidden] dtype: query, key and value
 *              blocks of n_heads * head_dim rows each (nn.Linear [out, in])
 *   w_qkv_gqa  [(n_heads + 2 * n_kv_heads) * head_dim, hidden] dtype, written;
 *              must not overlap w_qkv_mha
 *   hidden     a multiple of 8 (bf16) or 4 (fp32): rows are read as 16-byte
 *              vectors; both pointers 16-byte aligned
 * n_kv_heads = n_heads copies the weight; n_kv_heads = 1 gives MQA.
 * Errors: GQA_ERR_INVALID_ARG (null or overlapping buffers, non-positive
 * sizes, n_heads % n_kv_heads != 0), GQA_ERR_UNSUPPORTED_SHAPE (hidden not a
 * vector multiple), GQA_ERR_MISALIGNED, GQA_ERR_UNSUPPORTED_DTYPE, and the
 * device/launch statuses.  Asynchronous on `stream`; allocates nothing.
 */
int gqa_meanpool_kv_heads(const void* w_qkv_mha, int hidden, int n_heads, int n_kv_heads, int head_dim,
                          void* w_qkv_gqa, int dtype, void* stream);

/*
 * gqa_attn_decode_paged - gqa_attn_decode over a paged KV cache.
 *
 * Source: "MHA -> GQA: 提升 LLM 推理效率", section 3.2: a PagedAttention cache
 * keeps each sequence's keys and values in fixed-size pages that need not be
 * contiguous, and a block table lists a sequence's pages in order.  The
 * attention is exactly gqa_attn_decode over the cache that the table
 * describes; only the address of each key row changes.  Pages hold a whole
 * number of 64-key tiles, so every tile the kernel copies lies inside one
 * page and is fetched with one tensor copy per 64 columns, as in the
 * contiguous case.
 *
 *   q            [B, n_heads, head_dim] bf16
 *   k_pages,
 *   v_pages      [num_pages, n_kv_heads, page_size, head_dim] bf16: key t of
 *                sequence b is row t % page_size of page
 *                block_table[b][t / page_size], for every KV head
 *   block_table  [B, max_pages] int32, row-major; entries past a sequence's
 *                last page are not read.  An entry outside [0, num_pages)
 *                raises GQA_DEVERR_PAGE_RANGE and its keys read as zeros
 *   kv_lens      [B] int32: clamped to [0, max_pages * page_size]
 *                (GQA_DEVERR_KVLEN_RANGE)
 *   page_size    keys per page: a positive multiple of 64
 *   kv_split     as for gqa_attn_decode, with cache_cap = max_pages * page_size
 *   out          [B, n_heads, head_dim] bf16
 *   workspace    as for gqa_attn_decode: at least
 *                gqa_attn_decode_workspace_size(B, n_heads, n_kv_heads,
 *                head_dim, max_pages * page_size, kv_split) bytes, zero-filled
 *                before its first use
 *
 * bf16 with head_dim 64 or 128 only (GQA_ERR_UNSUPPORTED_DTYPE /
 * GQA_ERR_UNSUPPORTED_SHAPE otherwise).  Same statuses as gqa_attn_decode;
 * asynchronous on `stream`.
 */
int gqa_attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                          const int32_t* block_table, const int32_t* kv_lens, int B, int n_heads,
                          int n_kv_heads, int head_dim, int page_size, int max_pages, int num_pages,
                          int kv_split, void* out, void* workspace, size_t workspace_bytes, int dtype,
                          void* stream);

/*
 * gqa_fp8_quantize_qkv - FP8 (e4m3) inputs for gqa_attn_prefill_fp8, with
 * incoherent processing.
 *
 * Source: "FlashAttention-3" (together.ai summary), section "FP8低精度と
 * incoherent processing": FP8 doubles the tensor-core rate, but outlier
 * features inflate the rounding error; multiplying queries and keys by one
 * random orthogonal matrix, a Hadamard transform with random signs, spreads
 * the outliers over the features before quantising, and leaves every score
 * q.k unchanged.  Here M = H diag(signs) / sqrt(head_dim), H the Sylvester
 * Hadamard matrix; q and k rows become x M, v is not rotated.  Each tensor is
 * then scaled by 448 / amax (its largest magnitude after the rotation) and
 * rounded to e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
 * nearest, ties to even, saturating at 448).
 *
 *   q          [B, n_heads, S, head_dim] bf16
 *   k_cache,
 *   v_cache    [B, n_kv_heads, cache_cap, head_dim] bf16; rows at or beyond
 *              kv_lens[b] are not read (they may hold NaN)
 *   kv_lens    [B] int32, clamped to [0, cache_cap]
 *   signs      HOST array of head_dim values, each +1 or -1 (read during the
 *              call), or NULL for no rotation
 *   q8         [B, n_heads, S, head_dim] e4m3 codes, written
 *   k8         [B, n_kv_heads, cache_cap, head_dim] e4m3, written (rows at or
 *              beyond kv_len are zero)
 *   v8t        [B, n_kv_heads, head_dim, cache_cap] e4m3, written TRANSPOSED
 *              (per KV head, one row of cache_cap keys per feature; keys at
 *              or beyond kv_len are zero)
 *   amax       DEVICE float[3], written: the largest magnitude of the
 *              rotated q, the rotated k and v; tensor t's scale is
 *              amax[t] / 448 (a zero tensor has amax 0 and codes 0)
 *
 * head_dim 64 or 128; cache_cap a multiple of 16.  Asynchronous on `stream`
 * (a memset of amax and three kernels); allocates nothing.
 */
int gqa_fp8_quantize_qkv(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_lens, int B,
                         int S, int n_heads, int n_kv_heads, int head_dim, int cache_cap, const int8_t* signs,
                         void* q8, void* k8, void* v8t, float* amax, void* stream);

/*
 * gqa_attn_prefill_fp8 - gqa_attn_prefill on FP8 inputs: the tiled online
 * softmax with S = Q K^T and O = P V both on the tensor cores in e4m3
 * (tcgen05 kind::f8f6f4, float32 accumulation).  The probabilities P are
 * rounded to e4m3 for P V (offset by 2^4 so that values down to 2^-10 of a
 * row's maximum keep full e4m3 precision); the row sums use the unrounded
 * float32 probabilities.  Source as gqa_fp8_quantize_qkv and gqa_attn_prefill.
 *
 *   q8, k8, v8t, amax  as written by gqa_fp8_quantize_qkv (with or without
 *                      the rotation: scores are the same either way)
 *   kv_lens            [B] int32; queries sit at positions kv_len - S + s
 *   causal             nonzero: key t visible to a query at position p iff t <= p
 *   out                [B, S, n_heads, head_dim] bf16
 *
 * head_dim 128 only; cache_cap a multiple of 16.  Statuses as
 * gqa_attn_prefill; asynchronous on `stream`; allocates nothing.
 */
int gqa_attn_prefill_fp8(const void* q8, const void* k8, const void* v8t, const float* amax, const int32_t* kv_lens,
                         int B, int S, int n_heads, int n_kv_heads, int head_dim, int cache_cap, int causal, void* out,
                         void* stream);

/*
 * gqa_debug_inject_launch_failures - testing aid (host-side fault
 * injection): the next n compute calls (projection, prefill, decode,
 * mean-pool) that pass argument validation return GQA_ERR_LAUNCH_FAILED
 * without launching anything, as a failed launch would; later calls run
 * normally.  n = 0 clears pending injections; n < 0 is GQA_ERR_INVALID_ARG.
 */
int gqa_debug_inject_launch_failures(int n);

/*
 * gqa_debug_set_wait_limit_ns - testing aid for the bounded waits: every
 * pipeline wait in the library's kernels gives up after this many
 * nanoseconds (ns = 0 restores the default of 2 s), sets
 * GQA_DEVERR_WAIT_TIMEOUT, lets the copies and MMAs its CTA has in flight
 * land, frees its tensor memory and returns.  Applies to the current device
 * from the next launch on; synchronous (a host-to-device copy).
 */
int gqa_debug_set_wait_limit_ns(uint64_t ns);

/*
 * gqa_debug_skip_next_kv_tile - testing aid (a wait that runs out, made on
 * purpose): in the next gqa_attn_prefill call that takes the head_dim-64
 * bf16 tensor-core kernel, the first CTA's copy thread does not load key
 * tile `tile` (of 128 keys), so the waits for it run out after the wait
 * limit; the call still returns and later calls run normally.  tile = -1
 * disarms; tile < -1 is GQA_ERR_INVALID_ARG.
 */
int gqa_debug_skip_next_kv_tile(int tile);

/*
 * gqa_debug_exp2_poly - testing aid: evaluates, for n device floats x, the
 * polynomial 2^x that the prefill softmax can run on the FMA pipe (range
 * reduction to n + f with |f| <= 1/2, a degree-3 minimax fit of 2^f in
 * relative error, inputs below -125 clamped) into poly[i], and CUDA's
 * exp2f(x[i]) into ref[i].  Device pointers; asynchronous on `stream`.
 */
int gqa_debug_exp2_poly(const float* x, int n, float* poly, float* ref, void* stream);

/* Human-readable text of a gqa_status value (static storage). */
const char* gqa_status_string(int status);

/*
 * gqa_device_error - debugging aid: waits for the current device to finish,
 * copies the device error word (GQA_DEVERR_* bits accumulated by earlier
 * calls) to *bits and clears it.  Unlike every other call it synchronises.
 */
int gqa_device_error(int* bits);

/*
 * gqa_launch_count - number of kernels this library has launched in this
 * process (all devices, all streams).  A host-side counter: reading it does
 * not touch the device.
 */
uint64_t gqa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_B200_H */
