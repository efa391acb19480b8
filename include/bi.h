/*
 * bi.h — batch-invariant forward-pass kernels for transformer inference (B200, sm_100a).
 *
 * What "batch-invariant" means here: the bits of any output row depend only on
 * that row's own inputs. They do not depend on how many rows were batched with it,
 * on its position in the batch, on the other rows, on how many SMs were free, or
 * on whether its keys/values were written to the cache earlier or in the current
 * chunk. Every kernel reduces each row in one fixed order, fixed by the problem's
 * static shape (K, N, D, head counts) and never by the batch size M, the number of
 * sequences B or their lengths. Sources:
 *   - "Defeating Nondeterminism in LLM Inference" technical summary (mobiles-han
 *     blog), section 対応策：バッチ不変なカーネル設計: the kernel table (RMSNorm uses a
 *     data-parallel strategy; MatMul uses one kernel configuration for all shapes;
 *     Attention joins cache and current tokens into one layout and uses fixed-size
 *     KV splits).
 *   - Techzine, "Thinking Machines wil AI voorspelbaarder maken": reductions and
 *     sums always happen in one fixed order, whatever the batch size or load.
 *   - hakusoku, "LLM推論における非決定性の克服", section カーネル実装と加算順序: no
 *     atomic adds in the forward pass; tree reductions give deterministic results.
 *   - "Greedy Decoding Is Not Precision-Invariant" (arXiv 2609.26621), abstract:
 *     greedy argmax with an FP32 recompute of the LM head only when the top-2
 *     logit margin is below a threshold.
 *
 * Conventions for every call:
 *   - bf16 tensors are raw bfloat16 bits (bi_bf16). All pointers except the
 *     workspace-size queries' are DEVICE pointers owned by the caller; the
 *     library never frees or keeps them.
 *   - Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy default
 *     stream) and never synchronise. Host validation runs first: on any error
 *     status nothing is launched.
 *   - Leading dimensions are in elements. bf16 pointers and leading dimensions
 *     must give 16-byte aligned rows (pointer % 16 == 0, ld % 8 == 0), else
 *     BI_ERR_ALIGN.
 *   - A launch failure returns BI_ERR_CUDA. Conditions only the device can see
 *     (a page id outside the store, a length beyond the page table, a bounded
 *     device wait that expired) set a device error word that
 *     bi_get_device_error() reads; the affected rows are skipped or zeroed.
 *   - No atomics touch any value; results are bit-identical run to run.
 *   - The library allocates no device memory: scratch space is a caller-owned
 *     workspace whose size the *_workspace_size() queries give.
 */
#ifndef BI_H_
#define BI_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t bi_bf16; /* raw bfloat16 bits */

typedef enum {
  BI_OK = 0,
  BI_ERR_NULL = 1,           /* a required pointer is NULL */
  BI_ERR_SHAPE = 2,          /* a size is negative, zero where not allowed, or inconsistent */
  BI_ERR_ALIGN = 3,          /* a pointer or leading dimension breaks the 16-byte rule */
  BI_ERR_WORKSPACE = 4,      /* workspace NULL or smaller than the size query */
  BI_ERR_UNSUPPORTED = 5,    /* valid request this build does not implement (e.g. D not 64/128) */
  BI_ERR_CUDA = 6,           /* a CUDA runtime/driver call failed */
  BI_ERR_DEVICE_TIMEOUT = 7, /* reported by bi_get_device_error: a bounded device wait expired */
  BI_ERR_DEVICE_INDEX = 8    /* reported by bi_get_device_error: a page id / seq id / length out of range */
} bi_status;

/* Human-readable name of a status code. Never NULL. */
const char* bi_status_string(int status);

/* ABI version of this library (increments on any signature change). */
int bi_version(void);

/* Compile-time constants of the invariant schedule. */
#define BI_PAGE_TOKENS 16   /* tokens per KV page */
#define BI_KV_SPLIT 256     /* tokens per attention split (fixed size, not a fixed count) */
#define BI_GEMM_BM 128      /* matmul tile rows per CTA (tcgen05 M); see bi_matmul_tile_m */
#define BI_GEMM_BN_MAX 256  /* widest matmul tile (tcgen05 N); see bi_matmul_tile_n */
#define BI_GEMM_BK 64       /* matmul K block; K is summed block by block in ascending order */

/*
 * RMSNorm. Source: "Defeating Nondeterminism in LLM Inference" summary, kernel
 * table, row RMSNorm (data-parallel: each row reduced alone, never split across
 * CTAs at small batch).
 *   y[m, k] = bf16_rne( x[m, k] * rsqrt( (sum_k x[m, k]^2) / K + eps ) * w[k] )
 * x: [M, K] bf16 row-major, row stride ldx. w: [K] bf16. y: [M, K] bf16, stride ldy
 * (y may alias x when ldy == ldx). fp32 accumulation in one fixed order per row
 * that depends on K only. M == 0 is a no-op. Requires 8 <= K <= 16384, K % 8 == 0.
 */
bi_status bi_rmsnorm(const bi_bf16* x, int64_t ldx, const bi_bf16* w, bi_bf16* y, int64_t ldy,
                     int64_t M, int64_t K, float eps, void* stream);

/*
 * MatMul, C = A * W^T. Source: same table, row MatMul (one kernel configuration
 * for every shape; no split-K; no switching between tensor-core and other paths).
 *   C[m, n] = bf16_rne( sum_k A[m, k] * W[n, k] ),  fp32 accumulation in TMEM
 * A: [M, K] bf16 row-major (K contiguous), stride lda. W: [N, K] bf16 row-major
 * (the nn.Linear weight layout), stride ldw. C: [M, N] bf16, stride ldc; must not
 * overlap A or W. Each C[m, n] is one chain of tcgen05.mma instructions (bf16
 * operands, fp32 accumulator in tensor memory; 16 k each) over k = 0, 16, 32, ...
 * in ascending order, then one bf16 rounding; no split-K. That chain is the same
 * for every M and every position of the row or column inside its tile. The tile
 * (bi_matmul_tile_m rows: 128 on one SM, or 256 on a pair of SMs issuing
 * tcgen05.mma.cta_group::2; bi_matmul_tile_n columns) only decides how rows and
 * columns are dealt out to SMs and does not enter an element's arithmetic: the GPU
 * tests check that every row of every M in 1..2048 equals the same row of the
 * 2048-row product, bit for bit, across the tiles the sweep uses.
 * M == 0 or N == 0 is a no-op. Requires K % 64 == 0, K >= 64, N % 8 == 0.
 */
bi_status bi_matmul(const bi_bf16* A, int64_t lda, const bi_bf16* W, int64_t ldw, bi_bf16* C,
                    int64_t ldc, int64_t M, int64_t N, int64_t K, void* stream);

/*
 * Several products with the same A in one call: C_g = A * W_g^T for g = 0 .. count-1,
 * each exactly as bi_matmul would compute it (bit for bit: the same MMA chain per
 * element). A, M, K, lda as for bi_matmul; W, ldw, C, ldc, N: host arrays of count
 * entries (read before the call returns), each entry with bi_matmul's requirements;
 * no C_g may overlap A, any W_h or another C_h. 1 <= count <= BI_MATMUL_MULTI_MAX.
 * When every product would run on CTA-pair tiles alone (bi_matmul_tile_m == 256), one
 * launch takes the tiles of all of them in one list, so the SMs run whole rounds over
 * the joint list instead of a short last round per product; otherwise the products
 * are launched one after another. M == 0 is a no-op; a product with N == 0 is skipped.
 */
#define BI_MATMUL_MULTI_MAX 3
bi_status bi_matmul_multi(const bi_bf16* A, int64_t lda, int count, const bi_bf16* const* W, const int64_t* ldw,
                          bi_bf16* const* C, const int64_t* ldc, const int64_t* N, int64_t M, int64_t K,
                          void* stream);

/*
 * Tile width (32, 64, 128, 192 or 256 columns) that bi_matmul uses for an M x N
 * product on the current device; -1 if the device cannot be queried or M, N < 0.
 * Narrow tiles spread a small-M product over more SMs (each streams a thin slice
 * of W); wide tiles reuse each block of A for more columns at large M. The choice
 * follows the tile counts and the SM count; it changes which CTA computes a
 * column, never how. Host only, launches nothing.
 */
int bi_matmul_tile_n(int64_t M, int64_t N);

/*
 * Tile rows that bi_matmul uses for an M x N product on the current device: 128 (one
 * CTA per tile) or 256 (a cluster of two CTAs per tile, from M = 129 on where the
 * single-CTA tile would be 192 or 256 wide; each CTA loads half of the tile's A rows
 * and half of its W rows, and one tcgen05.mma.cta_group::2 covers both). -1 if the
 * device cannot be queried or M, N < 0. Host only, launches nothing.
 */
int bi_matmul_tile_m(int64_t M, int64_t N);

/*
 * Workspace bytes for bi_attention_decode (rows = B) or bi_attention_prefill
 * (rows = T). Depends on rows, Hq, D and the page-table width only.
 */
size_t bi_attention_workspace_size(int64_t rows, int Hq, int D, int max_pages_per_seq);

/*
 * Decode attention over the unified paged KV store. Source: same table, row
 * Attention (cache and current tokens in one layout; fixed-size KV splits), and
 * the FixedAttention sketch in the usage article, section 注意点・補足実装.
 *   out[b, h, :] = softmax_j( scale * q[b, h, :] . K_b[j, g, :] ) V_b[j, g, :],
 *   j = 0 .. seq_lens[b]-1, g = h / (Hq / Hkv).
 * q: [B, Hq, D] bf16. k_cache, v_cache: [num_pages, Hkv, 16, D] bf16 (a page holds
 * 16 consecutive tokens of one sequence for every kv-head). page_table: [B,
 * max_pages_per_seq] int32; token j of sequence b is slot j % 16 of physical page
 * page_table[b, j / 16]; entries past the last page are never read. seq_lens: [B]
 * int32. out: [B, Hq, D] bf16. Schedule: tokens are cut into splits at absolute
 * positions 0, 256, 512, ... (split count grows with the length); each split is
 * reduced over its 16-token pages in order, then splits are folded in ascending
 * order. Slots past a sequence's length are never read into the result (stale
 * pages may hold NaN). A sequence of length 0 yields zeros. D in {64, 128};
 * Hq % Hkv == 0 and Hq / Hkv in {1, 2, 4, 8}. workspace: >= the size query.
 */
bi_status bi_attention_decode(const bi_bf16* q, const bi_bf16* k_cache, const bi_bf16* v_cache,
                              int64_t num_pages, const int32_t* page_table, int max_pages_per_seq,
                              const int32_t* seq_lens, bi_bf16* out, int B, int Hq, int Hkv, int D,
                              float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode attention for callers that cannot allocate device memory. The pages have
 * no counterpart for this call; it exists for code that may not call cudaMalloc or
 * hold an allocator: for example a plugin or callback running inside another
 * framework that owns every byte of device memory and forbids allocation there, or a
 * latency-critical path where cudaMalloc's implicit device-wide synchronisation is
 * not allowed.
 * Same arguments, result and schedule as bi_attention_decode (bit-identical
 * output), minus the workspace: the scratch is a fixed array of
 * BI_STATIC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits. A request whose workspace size
 * (bi_attention_workspace_size(B, Hq, D, max_pages_per_seq)) exceeds it returns
 * BI_ERR_WORKSPACE and launches nothing.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any stream
 *     capture.
 *   - All calls share the one array and it keeps the previous call's contents.
 *     Nothing in it needs to start at zero: every byte a call reads was written
 *     earlier in the same call. Calls that overlap on the GPU (different streams,
 *     or different host threads on the same device) race on the array and must be
 *     serialised by the caller.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
#define BI_STATIC_SCRATCH_BYTES ((size_t)32 << 20) /* 32 MiB */
bi_status bi_attention_decode_static(const bi_bf16* q, const bi_bf16* k_cache, const bi_bf16* v_cache,
                                     int64_t num_pages, const int32_t* page_table, int max_pages_per_seq,
                                     const int32_t* seq_lens, bi_bf16* out, int B, int Hq, int Hkv, int D,
                                     float scale, void* stream);

/*
 * Causal prefill attention over the same store (chunked or whole). Source: same
 * table, row Attention (chunked prefill / prefix caching must not change the
 * path), and the usage article's test list (prefill, decode, cache on or off).
 * Query row t belongs to sequence q_seq[t] at absolute position q_pos[t] and sees
 * that sequence's keys 0 .. q_pos[t] (inclusive). The chunk's own K/V must already
 * be in the store (bi_kv_append), so cached and fresh tokens take one code path.
 * Each row is computed with exactly the per-row schedule of bi_attention_decode
 * for length q_pos[t] + 1, so a row's bits do not depend on the chunking, on T,
 * or on which other rows are present, and equal the decode result at that length.
 * A batch may therefore mix prefill chunks and decode tokens (a decode token is a
 * row at its sequence's newest position).
 * q: row t at q + t * ldq holds [Hq, D] bf16 (ldq >= Hq*D, ldq % 8 == 0, e.g. the
 * q part of a fused QKV projection). q_seq, q_pos: [T] int32. page_table:
 * [num_seqs, max_pages_per_seq] int32. out: [T, Hq, D] bf16. T == 0 is a no-op.
 */
bi_status bi_attention_prefill(const bi_bf16* q, int64_t ldq, const int32_t* q_seq, const int32_t* q_pos,
                               const bi_bf16* k_cache, const bi_bf16* v_cache, int64_t num_pages,
                               const int32_t* page_table, int num_seqs, int max_pages_per_seq,
                               bi_bf16* out, int T, int Hq, int Hkv, int D, float scale,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Causal prefill of one chunk on tensor cores (tcgen05). Source: same table, row
 * Attention, and the French article's section on the price of bit-identical output
 * (a faster attention kernel brought 55 s back to 42 s). The query rows are
 * positions pos0 .. pos0+T-1 of sequence `seq`; row t of q starts at q + t * ldq
 * and holds [Hq, D] bf16; the chunk's own K/V must already be in the store.
 * out: [T, Hq, D] bf16. Per row: keys in blocks of 64 at absolute positions,
 * ascending; S = q.k by tcgen05 (fp32), online softmax in fp32 by one thread per
 * row, P rounded to bf16, O += P V by tcgen05; out = O / l. A row's bits depend on
 * its position and the keys only, so whole and chunked prefill give the same bits.
 * They are NOT the bits of bi_attention_prefill / bi_attention_decode (a different,
 * also fixed, arithmetic; the two agree within the bf16 tolerance).
 * D in {64, 128} and Hq / Hkv even (two query heads of one kv-head share each
 * K/V block), else BI_ERR_UNSUPPORTED; scale > 0; pos0 + T <= max_pages_per_seq * 16.
 * No workspace.
 */
bi_status bi_attention_prefill_tc(const bi_bf16* q, int64_t ldq, int seq, int pos0, int T, const bi_bf16* k_cache,
                                  const bi_bf16* v_cache, int64_t num_pages, const int32_t* page_table, int num_seqs,
                                  int max_pages_per_seq, bi_bf16* out, int Hq, int Hkv, int D, float scale,
                                  void* stream);

/*
 * Glue: write new tokens' K/V into the paged store (the unified layout of the
 * FixedAttention sketch). Row t of k_new / v_new starts at t * ld_new and holds
 * [Hkv, D] bf16 (ld_new >= Hkv*D, ld_new % 8 == 0, e.g. the k / v parts of a fused
 * QKV projection); it goes to slot q_pos[t] % 16 of page
 * page_table[q_seq[t], q_pos[t] / 16]. Pure copies; T == 0 is a no-op.
 * Out-of-range ids set the device error word and skip the token.
 */
bi_status bi_kv_append(const bi_bf16* k_new, const bi_bf16* v_new, int64_t ld_new, const int32_t* q_seq,
                       const int32_t* q_pos, bi_bf16* k_cache, bi_bf16* v_cache, int64_t num_pages,
                       const int32_t* page_table, int num_seqs, int max_pages_per_seq, int T,
                       int Hkv, int D, void* stream);

/*
 * Glue of a Llama-style decoder step. Each output element depends only on its own
 * row's inputs (copies and elementwise fp32 math), so these are batch-invariant by
 * construction; they keep a whole decoder step inside this library between the
 * reductions above. No page describes them; they are the plain Llama operations.
 *
 * bi_gather_rows: dst[m, :width] = src[idx[m], :width] (embedding lookup, row
 *   selection). idx out of [0, nrows_src) sets the device error word and zeroes
 *   the row. width % 8 == 0.
 * bi_rope: rotary position embedding, rotate-half form, in place on the H heads of
 *   D dims in each row t of x (row stride ldx): for i < D/2 with
 *   (c, s) = cos_sin[2 * (pos[t] * D/2 + i) .. +1] (fp32, [max_pos][D/2][2]),
 *   x[i] <- x[i] c - x[i+D/2] s,  x[i+D/2] <- x[i+D/2] c + x[i] s, in fp32 as
 *   fma(a, c, -(b s)) and fma(b, c, a s), rounded to bf16.
 * bi_swiglu: out[m, j] = bf16(silu(g) * u), g = gate_up[m, j], u = gate_up[m, F+j],
 *   silu(g) = g / (1 + exp(-g)) in fp32. F % 8 == 0.
 * bi_add: out = bf16(a + b) elementwise over n (n % 8 == 0); out may alias a or b.
 */
bi_status bi_gather_rows(const bi_bf16* src, int64_t ld_src, int64_t nrows_src, const int32_t* idx, int64_t M,
                         int64_t width, bi_bf16* dst, int64_t ld_dst, void* stream);
bi_status bi_rope(bi_bf16* x, int64_t ldx, int64_t T, int H, int D, const int32_t* pos, const float* cos_sin,
                  int max_pos, void* stream);
bi_status bi_swiglu(const bi_bf16* gate_up, int64_t ld_gu, bi_bf16* out, int64_t ld_out, int64_t M, int64_t F,
                    void* stream);
bi_status bi_add(const bi_bf16* a, const bi_bf16* b, bi_bf16* out, int64_t n, void* stream);

/* Workspace bytes for bi_lmhead_argmax with M rows and vocabulary V. */
size_t bi_lmhead_workspace_size(int64_t M, int64_t V);

/*
 * Greedy LM head with selective FP32 recompute. Source: "Greedy Decoding Is Not
 * Precision-Invariant" (arXiv 2609.26621), abstract.
 *   1. logits = bi_matmul(h, W) rounded to bf16 (the first, bf16 pass);
 *   2. per row: top-2 of the bf16 logits (lowest index wins ties; NaN never
 *      wins), margin = top1 - top2 in fp32;
 *   3. rows with margin < margin_threshold are recomputed in fp32: operands
 *      widened from bf16, one fp32 FMA chain per logit in ascending k (no tensor
 *      cores, no TF32), and the token is the argmax of those fp32 logits;
 *      other rows keep the first-pass argmax.
 * h: [M, K] bf16, stride ldh. W: [V, K] bf16 contiguous. tokens: [M] int32 out.
 * recomputed: [M] int32 out (1 if the row took step 3, else 0). logits_fp32:
 * optional [M, V] fp32 out (may be NULL): rows that took step 3 receive their fp32
 * logits, other rows are not written. Requires the bi_matmul rules on K and
 * V % 8 == 0. M == 0 is a no-op.
 * How step 3 is laid out (never the arithmetic of a logit): with K <= 4096 it reads W
 * once for a single flagged row, once per group of 8 rows for 2..24 flagged rows, and
 * uses 64-row tiles beyond that; the choice is made on the device from the flagged
 * count. Every fp32 logit is the same FMA chain on every path (tested bit for bit).
 */
bi_status bi_lmhead_argmax(const bi_bf16* h, int64_t ldh, const bi_bf16* W, int64_t M, int64_t V,
                           int64_t K, float margin_threshold, int32_t* tokens, int32_t* recomputed,
                           float* logits_fp32, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * Row reductions for log-probabilities and means, and temperature sampling.
 * Source: "Defeating Nondeterminism" summary, section 他の演算子 (RMSNorm, MatMul,
 * mean/reduction etc.): log_softmax and mean get batch-invariant kernels too, a
 * mean reduced in one fixed order. Techzine, "Thinking Machines wil AI
 * voorspelbaarder maken": sampling and training bit-identical (on-policy RL).
 * One CTA per row; each row is reduced in one fixed order that depends on the row
 * length only (256 threads, each folding its 8-element vectors t, t+256, ... in
 * order; xor-butterfly inside a warp; the 8 warp values left to right), so a row's
 * result is the same bits whatever M and the other rows are.
 * Inputs are bf16 [M, N] rows (16-byte aligned, ld % 8 == 0, N % 8 == 0,
 * 8 <= N <= 2^24); M == 0 is a no-op. Rows of up to 32768 elements are read from
 * HBM once; longer rows are re-read per pass from L2 in the same order.
 */

/* y[m, i] = x[m, i] - lse_m with lse_m = max_m + log(sum_i exp(x[m, i] - max_m)),
 * the sum in fp32 in the order above (exp as 2^(x log2 e - max log2 e), one FMA and
 * the SFU exp2). y: [M, N] fp32, stride ldy (ldy % 4 == 0, 16-byte aligned). */
bi_status bi_log_softmax(const bi_bf16* x, int64_t ldx, float* y, int64_t ldy, int64_t M, int64_t N,
                         void* stream);

/* out[m] = x[m, tokens[m]] - lse_m (the same lse_m as bi_log_softmax): the
 * log-probability of each row's token. tokens: [M] int32 device; a token outside
 * 0..N-1 gives NaN and BI_ERR_DEVICE_INDEX in the device error word. out: [M] fp32. */
bi_status bi_token_logprob(const bi_bf16* x, int64_t ldx, const int32_t* tokens, float* out, int64_t M,
                           int64_t N, void* stream);

/* y[m] = (sum_k x[m, k]) / K, the sum in fp32 in the order above, one division. y: [M] fp32. */
bi_status bi_row_mean(const bi_bf16* x, int64_t ldx, float* y, int64_t M, int64_t K, void* stream);

/*
 * The uniforms the sampler draws: u[m, i] in (0, 1) for vocabulary entry i of row m,
 * from Philox4x64-10 (Salmon et al., "Parallel random numbers: as easy as 1, 2, 3",
 * SC 2011) with key (seeds[m], 0) and counter (i / 8, steps[m], 0, 0): entry i takes
 * output word (i % 8) / 2, its low 32 bits for even i and its high 32 bits for odd i,
 * and u = (top 23 of those 32 bits + 1/2) * 2^-23 (exact in fp32). A row's draws depend on
 * (seed, step, i) only: the request's seed and its decode step, never the batch.
 * seeds, steps: [M] uint64 device. u: [M, V] fp32, stride ldu (ldu % 4 == 0).
 */
bi_status bi_sampling_uniforms(const uint64_t* seeds, const uint64_t* steps, float* u, int64_t ldu, int64_t M,
                               int64_t V, void* stream);

/*
 * Temperature sampling by the Gumbel-max rule: tokens[m] = argmax_i
 * fma(x[m, i], 1/T, g_i) in fp32 with g_i = -log(-log u[m, i]) (the uniforms of
 * bi_sampling_uniforms) and 1/T rounded once; lowest index among equal scores. A
 * draw from softmax(x / T) that depends on (logits, seed, step) only. logits: [M, V]
 * bf16 (e.g. the bi_matmul LM-head output); temperature: finite, > 0; tokens: [M]
 * int32 out. A row whose scores are all NaN gives token 0 and BI_ERR_DEVICE_INDEX.
 * Each row runs on a cluster of 8 CTAs, each taking a fixed eighth of the vocabulary
 * (the argmax is exact, so the split does not change the token).
 */
bi_status bi_sample(const bi_bf16* logits, int64_t ld, const uint64_t* seeds, const uint64_t* steps,
                    float temperature, int32_t* tokens, int64_t M, int64_t V, void* stream);

/*
 * Self-test of the device-side failure detection (no page describes it). Launches
 * one thread that waits on an mbarrier nothing will complete, using the same
 * bounded wait as every kernel here but a limit of limit_ms milliseconds (1..2000;
 * the kernels use 2000). When the limit expires the kernel records
 * BI_ERR_DEVICE_TIMEOUT in the device error word and returns, so the context stays
 * usable. Returns BI_ERR_SHAPE for a limit outside 1..2000.
 */
bi_status bi_selftest_wait_timeout(int limit_ms, void* stream);

/*
 * Reads and clears the device error word of the current device (synchronises the
 * device first). *code receives BI_OK, BI_ERR_DEVICE_TIMEOUT or
 * BI_ERR_DEVICE_INDEX (the first error recorded since the last read). Returns
 * BI_ERR_NULL if code is NULL, BI_ERR_CUDA if the read fails.
 */
bi_status bi_get_device_error(int32_t* code);

#ifdef __cplusplus
}
#endif

#endif /* BI_H_ */
