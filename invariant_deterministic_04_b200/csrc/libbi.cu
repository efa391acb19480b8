// libbi: the C ABI of the batch-invariant kernels (declared in include/bi.h).
//
// One translation unit: the kernels are included here so that they share the
// device error word without relocatable device code. Every entry point validates
// its arguments on the host first and launches nothing on error.
#include <climits>
#include <cmath>
#include <mutex>

#include "device.cuh"
#include "rmsnorm.cuh"
#include "gemm.cuh"
#include "attention.cuh"
#include "lmhead.cuh"
#include "glue.cuh"
#include "attention_tc.cuh"
#include "reduce.cuh"

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t n) { return (n + 255) & ~size_t(255); }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bool ranges_overlap(const void* a, size_t abytes, const void* b, size_t bbytes) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bbytes && b0 < a0 + abytes;
}

size_t span_bytes(int64_t rows, int64_t cols, int64_t ld, size_t elem) {
  return rows <= 0 ? 0 : (size_t)((rows - 1) * ld + cols) * elem;
}

// Whether two M-row blocks of 2-byte elements (rows of na / nb elements, lda / ldb
// elements apart, na <= lda, nb <= ldb) share an element. Exact for equal row strides,
// where column ranges of one wider matrix are disjoint: elements a + i*ld + j and
// b + i'*ld + j' coincide iff (i - i')*ld + (j - j') = (b - a), and with both widths at
// most ld only k = i - i' = floor((b - a) / ld) and k + 1 can give j - j' in (-nb, na).
// Otherwise by the blocks' address spans.
bool blocks_overlap(const void* a, int64_t lda, int64_t na, const void* b, int64_t ldb, int64_t nb, int64_t M) {
  if (M <= 0 || na <= 0 || nb <= 0) return false;
  const int64_t db = (int64_t)(reinterpret_cast<intptr_t>(b) - reinterpret_cast<intptr_t>(a));
  if (lda != ldb || db % 2 != 0) return ranges_overlap(a, span_bytes(M, na, lda, 2), b, span_bytes(M, nb, ldb, 2));
  const int64_t d = db / 2;
  const int64_t k0 = d >= 0 ? d / lda : -((-d + lda - 1) / lda);
  for (int64_t k = k0; k <= k0 + 1; ++k) {
    if (k <= -M || k >= M) continue;
    const int64_t r = d - k * lda;
    if (r > -nb && r < na) return true;
  }
  return false;
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// ---- attention helpers

int max_splits(int max_pages_per_seq) { return (max_pages_per_seq + bi::attn::PAGES_PER_SPLIT - 1) / bi::attn::PAGES_PER_SPLIT; }

struct AttnWs {
  int32_t* off;
  float2* pml;
  float* po;
};

size_t attn_ws_size(int64_t rows, int Hq, int D, int max_pages, AttnWs* layout, void* base) {
  if (rows < 0 || Hq <= 0 || D <= 0 || max_pages <= 0) return 0;
  const int64_t ms = max_splits(max_pages);
  const size_t off_b = align256((size_t)(rows + 1) * 4);
  const size_t pml_b = align256((size_t)rows * ms * Hq * 8);
  const size_t po_b = align256((size_t)rows * ms * Hq * D * 4);
  if (layout && base) {
    uint8_t* p = static_cast<uint8_t*>(base);
    layout->off = reinterpret_cast<int32_t*>(p);
    layout->pml = reinterpret_cast<float2*>(p + off_b);
    layout->po = reinterpret_cast<float*>(p + off_b + pml_b);
  }
  return off_b + pml_b + po_b;
}

template <int D, int G>
cudaError_t launch_split(const uint16_t* q, int64_t ldq, int Hq, int Hkv, const uint16_t* kc,
                         const uint16_t* vc, int64_t num_pages, const int32_t* pt, bi::attn::Rows R, int nrows,
                         const AttnWs& ws, float c, cudaStream_t st) {
  constexpr int smem = bi::attn::split_smem_bytes<D, G>();
  constexpr int threads = bi::attn::SplitCfg<D, G>::WARPS * 32;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  // the shared-memory limit and the occupancy query run once per device; their
  // result is kept, so a failure is returned on every later call as well
  static std::once_flag once[64];
  static cudaError_t result[64];
  static int per_sm[64];
  std::call_once(once[dev], [&] {
    cudaError_t e = cudaFuncSetAttribute(bi::attn::attn_split_kernel<D, G>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm[dev], bi::attn::attn_split_kernel<D, G>, threads,
                                                        smem);
    if (e == cudaSuccess && per_sm[dev] <= 0) e = cudaErrorInvalidConfiguration;
    result[dev] = e;
  });
  if (result[dev] != cudaSuccess) return result[dev];
  // persistent grid: as many CTAs as can be resident (shared memory or registers
  // limit it); the grid only decides which warp takes which (row, head, split)
  const int grid = device_sms() * per_sm[dev];
  return bi::launch_pdl(bi::attn::attn_split_kernel<D, G>, dim3(grid), dim3(threads), (size_t)smem, st, q, ldq, Hq, Hkv,
                    kc, vc, num_pages, pt, R, nrows, (const int32_t*)ws.off, ws.po, ws.pml, c);
}

template <int D>
cudaError_t launch_split_g(int G, const uint16_t* q, int64_t ldq, int Hq, int Hkv, const uint16_t* kc, const uint16_t* vc,
                           int64_t num_pages, const int32_t* pt, bi::attn::Rows R, int nrows, const AttnWs& ws,
                           float c, cudaStream_t st) {
  switch (G) {
    case 1: return launch_split<D, 1>(q, ldq, Hq, Hkv, kc, vc, num_pages, pt, R, nrows, ws, c, st);
    case 2: return launch_split<D, 2>(q, ldq, Hq, Hkv, kc, vc, num_pages, pt, R, nrows, ws, c, st);
    case 4: return launch_split<D, 4>(q, ldq, Hq, Hkv, kc, vc, num_pages, pt, R, nrows, ws, c, st);
    default: return launch_split<D, 8>(q, ldq, Hq, Hkv, kc, vc, num_pages, pt, R, nrows, ws, c, st);
  }
}

// Host checks of an attention request that need no workspace: head counts, head
// size, scale, strides, the 32-bit range of the work list, pointer alignment.
bi_status attention_check(const uint16_t* q, int64_t ldq, const uint16_t* kc, const uint16_t* vc, int64_t num_pages,
                          int max_pages, int nrows, const uint16_t* out, int Hq, int Hkv, int D, float scale) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || num_pages <= 0 || max_pages <= 0) return BI_ERR_SHAPE;
  const int G = Hq / Hkv;
  if ((D != 64 && D != 128) || (G != 1 && G != 2 && G != 4 && G != 8)) return BI_ERR_UNSUPPORTED;
  if (!std::isfinite(scale) || ldq < (int64_t)Hq * D) return BI_ERR_SHAPE;
  if (ldq % 8) return BI_ERR_ALIGN;
  // index arithmetic of the work list is 32-bit
  if ((int64_t)nrows * max_splits(max_pages) * Hkv >= INT_MAX || (int64_t)nrows * Hq >= INT_MAX / 8)
    return BI_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(out)) return BI_ERR_ALIGN;
  return BI_OK;
}

bi_status attention_common(const uint16_t* q, int64_t ldq, const uint16_t* kc, const uint16_t* vc, int64_t num_pages,
                           const int32_t* pt, int max_pages, bi::attn::Rows R, int nrows, uint16_t* out,
                           int Hq, int Hkv, int D, float scale, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (bi_status e = attention_check(q, ldq, kc, vc, num_pages, max_pages, nrows, out, Hq, Hkv, D, scale)) return e;
  if (!aligned16(ws)) return BI_ERR_ALIGN;
  const int G = Hq / Hkv;
  AttnWs lay{};
  const size_t need = attn_ws_size(nrows, Hq, D, max_pages, &lay, ws);
  if (ws_bytes < need) return BI_ERR_WORKSPACE;
  if (nrows == 0) return BI_OK;
  const float c = (float)((double)scale * 1.4426950408889634);  // scale * log2(e)
  if (bi::launch_pdl(bi::attn::split_offsets_kernel, dim3(1), dim3(1024), 0, st, R, nrows, lay.off) != cudaSuccess)
    return BI_ERR_CUDA;
  cudaError_t e = D == 128 ? launch_split_g<128>(G, q, ldq, Hq, Hkv, kc, vc, num_pages, pt, R, nrows, lay, c, st)
                           : launch_split_g<64>(G, q, ldq, Hq, Hkv, kc, vc, num_pages, pt, R, nrows, lay, c, st);
  if (e != cudaSuccess) return BI_ERR_CUDA;
  // one dim per lane while that still leaves at most 32 warps per SM; beyond that
  // D / 32 dims per lane (fewer, wider loads). The fold is the same either way.
  const int sms = device_sms();
  if (sms <= 0) return BI_ERR_CUDA;
  const bool narrow = (int64_t)nrows * Hq * (D / 32) <= (int64_t)sms * 32;
  const int warps = narrow ? nrows * Hq * (D / 32) : nrows * Hq;
  const int grid = (warps + 7) / 8;
  if (D == 128) {
    if (narrow)
      e = bi::launch_pdl(bi::attn::attn_combine_kernel<128, 1>, dim3(grid), dim3(256), 0, st, (const float*)lay.po,
                     (const float2*)lay.pml, (const int32_t*)lay.off, nrows, Hq, out);
    else
      e = bi::launch_pdl(bi::attn::attn_combine_kernel<128, 4>, dim3(grid), dim3(256), 0, st, (const float*)lay.po,
                     (const float2*)lay.pml, (const int32_t*)lay.off, nrows, Hq, out);
  } else {
    if (narrow)
      e = bi::launch_pdl(bi::attn::attn_combine_kernel<64, 1>, dim3(grid), dim3(256), 0, st, (const float*)lay.po,
                     (const float2*)lay.pml, (const int32_t*)lay.off, nrows, Hq, out);
    else
      e = bi::launch_pdl(bi::attn::attn_combine_kernel<64, 2>, dim3(grid), dim3(256), 0, st, (const float*)lay.po,
                     (const float2*)lay.pml, (const int32_t*)lay.off, nrows, Hq, out);
  }
  return e == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

// ---- LM head workspace: bf16 logits [M, V], fp32 logits [M, V], flagged list [M + 1],
// argmax partials of the streaming recompute [24][its CTAs], its completion ticket
struct LmWs {
  uint16_t* logits16;
  float* logits32;
  int32_t* list;
  bi::lmhead::ArgBest* arg_part;
  unsigned int* ticket;
};

size_t lm_ws_size(int64_t M, int64_t V, LmWs* lay, void* base) {
  if (M < 0 || V <= 0) return 0;
  const int64_t sctas = (V + bi::lmhead::kStrWarps * 32 - 1) / (bi::lmhead::kStrWarps * 32);
  const size_t a = align256((size_t)M * V * 2), b = align256((size_t)M * V * 4), c = align256((size_t)(M + 1) * 4);
  const size_t d = align256((size_t)bi::lmhead::kStrMaxCount * sctas * sizeof(bi::lmhead::ArgBest)), e = 256;
  if (lay && base) {
    uint8_t* p = static_cast<uint8_t*>(base);
    lay->logits16 = reinterpret_cast<uint16_t*>(p);
    lay->logits32 = reinterpret_cast<float*>(p + a);
    lay->list = reinterpret_cast<int32_t*>(p + a + b);
    lay->arg_part = reinterpret_cast<bi::lmhead::ArgBest*>(p + a + b + c);
    lay->ticket = reinterpret_cast<unsigned int*>(p + a + b + c + d);
  }
  return a + b + c + d + e;
}

}  // namespace

// Scratch of bi_attention_decode_static: a fixed array instead of a caller
// workspace, for callers that cannot allocate device memory. Every GPU that loads
// the library holds it until the process exits. Host code may not pass the
// symbol itself to a kernel (on the host it names a stand-in, not device memory):
// its device address is looked up once per device below.
static __device__ __align__(256) unsigned char g_decode_scratch[BI_STATIC_SCRATCH_BYTES];

namespace {

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};

// Device address of g_decode_scratch on the current device (looked up on first use).
bi_status decode_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BI_ERR_CUDA;
  if (dev < 0 || dev >= 64) return BI_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return BI_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return BI_OK;
}

}  // namespace

extern "C" {

const char* bi_status_string(int status) {
  switch (status) {
    case BI_OK: return "BI_OK";
    case BI_ERR_NULL: return "BI_ERR_NULL";
    case BI_ERR_SHAPE: return "BI_ERR_SHAPE";
    case BI_ERR_ALIGN: return "BI_ERR_ALIGN";
    case BI_ERR_WORKSPACE: return "BI_ERR_WORKSPACE";
    case BI_ERR_UNSUPPORTED: return "BI_ERR_UNSUPPORTED";
    case BI_ERR_CUDA: return "BI_ERR_CUDA";
    case BI_ERR_DEVICE_TIMEOUT: return "BI_ERR_DEVICE_TIMEOUT";
    case BI_ERR_DEVICE_INDEX: return "BI_ERR_DEVICE_INDEX";
    default: return "BI_ERR_UNKNOWN";
  }
}

int bi_version(void) { return 4; }

bi_status bi_rmsnorm(const bi_bf16* x, int64_t ldx, const bi_bf16* w, bi_bf16* y, int64_t ldy, int64_t M,
                     int64_t K, float eps, void* stream) {
  if (!x || !w || !y) return BI_ERR_NULL;
  if (M < 0 || K < 8 || K % 8 != 0 || ldx < K || ldy < K || M > INT_MAX || !std::isfinite(eps) || eps < 0)
    return BI_ERR_SHAPE;
  if (K > 16384) return BI_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || ldx % 8 || ldy % 8) return BI_ERR_ALIGN;
  if (M == 0) return BI_OK;
  // in place only row for row: an alias with another row stride would let one row's
  // output overwrite another row's input before it is read
  if (x == y ? ldx != ldy : ranges_overlap(x, span_bytes(M, K, ldx, 2), y, span_bytes(M, K, ldy, 2)))
    return BI_ERR_SHAPE;
  const int sms = device_sms();
  if (sms <= 0) return BI_ERR_CUDA;
  return bi::rms::launch(x, ldx, w, y, ldy, M, (int)K, eps, sms, as_stream(stream)) == cudaSuccess ? BI_OK
                                                                                                   : BI_ERR_CUDA;
}

bi_status bi_matmul(const bi_bf16* A, int64_t lda, const bi_bf16* W, int64_t ldw, bi_bf16* C, int64_t ldc,
                    int64_t M, int64_t N, int64_t K, void* stream) {
  if (!A || !W || !C) return BI_ERR_NULL;
  if (M < 0 || N < 0 || K < 64 || K % 64 != 0 || N % 8 != 0 || M > INT_MAX || N > INT_MAX || K > INT_MAX)
    return BI_ERR_SHAPE;
  if (lda < K || ldw < K || ldc < N) return BI_ERR_SHAPE;
  if (!aligned16(A) || !aligned16(W) || !aligned16(C) || lda % 8 || ldw % 8 || ldc % 8) return BI_ERR_ALIGN;
  if (M == 0 || N == 0) return BI_OK;
  const size_t cb = span_bytes(M, N, ldc, 2);
  if (ranges_overlap(C, cb, A, span_bytes(M, K, lda, 2)) || ranges_overlap(C, cb, W, span_bytes(N, K, ldw, 2)))
    return BI_ERR_SHAPE;
  return bi::gemm::launch(A, lda, W, ldw, C, ldc, M, N, K, as_stream(stream));
}

bi_status bi_matmul_multi(const bi_bf16* A, int64_t lda, int count, const bi_bf16* const* W, const int64_t* ldw,
                          bi_bf16* const* C, const int64_t* ldc, const int64_t* N, int64_t M, int64_t K,
                          void* stream) {
  if (!A || !W || !ldw || !C || !ldc || !N) return BI_ERR_NULL;
  if (count < 1 || count > BI_MATMUL_MULTI_MAX) return BI_ERR_SHAPE;
  if (M < 0 || K < 64 || K % 64 != 0 || M > INT_MAX || K > INT_MAX || lda < K) return BI_ERR_SHAPE;
  if (!aligned16(A) || lda % 8) return BI_ERR_ALIGN;
  const size_t abytes = span_bytes(M, K, lda, 2);
  bi::gemm::Product prods[BI_MATMUL_MULTI_MAX];
  int live = 0;
  for (int g = 0; g < count; ++g) {
    if (!W[g] || !C[g]) return BI_ERR_NULL;
    if (N[g] < 0 || N[g] % 8 != 0 || N[g] > INT_MAX || ldw[g] < K || ldc[g] < N[g]) return BI_ERR_SHAPE;
    if (!aligned16(W[g]) || !aligned16(C[g]) || ldw[g] % 8 || ldc[g] % 8) return BI_ERR_ALIGN;
  }
  for (int g = 0; g < count; ++g) {
    if (M == 0 || N[g] == 0) continue;
    const size_t cb = span_bytes(M, N[g], ldc[g], 2);
    if (ranges_overlap(C[g], cb, A, abytes)) return BI_ERR_SHAPE;
    for (int h = 0; h < count; ++h) {
      if (N[h] > 0 && ranges_overlap(C[g], cb, W[h], span_bytes(N[h], K, ldw[h], 2))) return BI_ERR_SHAPE;
      if (h != g && blocks_overlap(C[g], ldc[g], N[g], C[h], ldc[h], N[h], M)) return BI_ERR_SHAPE;
    }
    prods[live++] = bi::gemm::Product{W[g], ldw[g], C[g], ldc[g], N[g]};
  }
  if (live == 0) return BI_OK;
  return bi::gemm::launch_multi(A, lda, prods, live, M, K, as_stream(stream));
}

int bi_matmul_tile_n(int64_t M, int64_t N) {
  if (M < 0 || N < 0) return -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  const int sms = bi::gemm::device_sms(dev);
  if (sms <= 0) return -1;
  const int pair = bi::gemm::pick_pair(M, N, sms);
  return pair ? pair : bi::gemm::pick_bn(M, N, sms);
}

int bi_matmul_tile_m(int64_t M, int64_t N) {
  if (M < 0 || N < 0) return -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  const int sms = bi::gemm::device_sms(dev);
  if (sms <= 0) return -1;
  return bi::gemm::pick_pair(M, N, sms) ? 256 : 128;
}

size_t bi_attention_workspace_size(int64_t rows, int Hq, int D, int max_pages_per_seq) {
  return attn_ws_size(rows, Hq, D, max_pages_per_seq, nullptr, nullptr);
}

bi_status bi_attention_decode(const bi_bf16* q, const bi_bf16* k_cache, const bi_bf16* v_cache, int64_t num_pages,
                              const int32_t* page_table, int max_pages_per_seq, const int32_t* seq_lens,
                              bi_bf16* out, int B, int Hq, int Hkv, int D, float scale, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!q || !k_cache || !v_cache || !page_table || !seq_lens || !out) return BI_ERR_NULL;
  if (B < 0) return BI_ERR_SHAPE;
  if (!workspace) return B == 0 ? BI_OK : BI_ERR_WORKSPACE;
  bi::attn::Rows R{seq_lens, nullptr, nullptr, B, max_pages_per_seq};
  return attention_common(q, (int64_t)Hq * D, k_cache, v_cache, num_pages, page_table, max_pages_per_seq, R, B, out,
                          Hq, Hkv, D, scale, workspace, workspace_bytes, as_stream(stream));
}

bi_status bi_attention_decode_static(const bi_bf16* q, const bi_bf16* k_cache, const bi_bf16* v_cache,
                                     int64_t num_pages, const int32_t* page_table, int max_pages_per_seq,
                                     const int32_t* seq_lens, bi_bf16* out, int B, int Hq, int Hkv, int D,
                                     float scale, void* stream) {
  if (!q || !k_cache || !v_cache || !page_table || !seq_lens || !out) return BI_ERR_NULL;
  if (B < 0) return BI_ERR_SHAPE;
  if (B == 0) return BI_OK;
  // every check that needs no scratch runs before the size check and before the
  // first use of the device (the symbol lookup)
  if (bi_status e = attention_check(q, (int64_t)Hq * D, k_cache, v_cache, num_pages, max_pages_per_seq, B, out, Hq,
                                    Hkv, D, scale))
    return e;
  if (attn_ws_size(B, Hq, D, max_pages_per_seq, nullptr, nullptr) > BI_STATIC_SCRATCH_BYTES) return BI_ERR_WORKSPACE;
  void* scratch = nullptr;
  const bi_status s = decode_scratch_address(&scratch);
  if (s != BI_OK) return s;
  bi::attn::Rows R{seq_lens, nullptr, nullptr, B, max_pages_per_seq};
  return attention_common(q, (int64_t)Hq * D, k_cache, v_cache, num_pages, page_table, max_pages_per_seq, R, B, out,
                          Hq, Hkv, D, scale, scratch, BI_STATIC_SCRATCH_BYTES, as_stream(stream));
}

bi_status bi_attention_prefill(const bi_bf16* q, int64_t ldq, const int32_t* q_seq, const int32_t* q_pos,
                               const bi_bf16* k_cache, const bi_bf16* v_cache, int64_t num_pages,
                               const int32_t* page_table, int num_seqs, int max_pages_per_seq, bi_bf16* out,
                               int T, int Hq, int Hkv, int D, float scale, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (!q || !q_seq || !q_pos || !k_cache || !v_cache || !page_table || !out) return BI_ERR_NULL;
  if (T < 0 || num_seqs <= 0) return BI_ERR_SHAPE;
  if (!workspace) return T == 0 ? BI_OK : BI_ERR_WORKSPACE;
  bi::attn::Rows R{nullptr, q_seq, q_pos, num_seqs, max_pages_per_seq};
  return attention_common(q, ldq, k_cache, v_cache, num_pages, page_table, max_pages_per_seq, R, T, out, Hq, Hkv, D,
                          scale, workspace, workspace_bytes, as_stream(stream));
}

bi_status bi_attention_prefill_tc(const bi_bf16* q, int64_t ldq, int seq, int pos0, int T, const bi_bf16* k_cache,
                                  const bi_bf16* v_cache, int64_t num_pages, const int32_t* page_table, int num_seqs,
                                  int max_pages_per_seq, bi_bf16* out, int Hq, int Hkv, int D, float scale,
                                  void* stream) {
  if (!q || !k_cache || !v_cache || !page_table || !out) return BI_ERR_NULL;
  if (T < 0 || pos0 < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || num_pages <= 0 || num_seqs <= 0 ||
      max_pages_per_seq <= 0 || seq < 0 || seq >= num_seqs || !std::isfinite(scale))
    return BI_ERR_SHAPE;
  if (D != 64 && D != 128 || (Hq / Hkv) % 2 != 0) return BI_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) return BI_ERR_SHAPE;
  if ((int64_t)pos0 + T > (int64_t)max_pages_per_seq * BI_PAGE_TOKENS || ldq < (int64_t)Hq * D) return BI_ERR_SHAPE;
  // the work list (128-row blocks x head pairs) is indexed in 32-bit
  if (((int64_t)T + bi::attn_tc::ROWS - 1) / bi::attn_tc::ROWS * (Hq / 2) >= INT_MAX / 2) return BI_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || ldq % 8) return BI_ERR_ALIGN;
  if (T == 0) return BI_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BI_ERR_CUDA;
  const int sms = bi::gemm::device_sms(dev);
  if (sms <= 0) return BI_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  const int64_t kv_rows = num_pages * Hkv * BI_PAGE_TOKENS;
  if (!bi::gemm::make_map(&tq, q, T, (int64_t)Hq * D, ldq, bi::attn_tc::ROWS) ||
      !bi::gemm::make_map(&tk, k_cache, kv_rows, D, D, BI_PAGE_TOKENS) ||
      !bi::gemm::make_map(&tv, v_cache, kv_rows, D, D, BI_PAGE_TOKENS))
    return BI_ERR_CUDA;
  // one work item = two query heads of one kv-head over one 128-row block
  const int work = ((T + bi::attn_tc::ROWS - 1) / bi::attn_tc::ROWS) * (Hq / 2);
  const int grid = work < sms ? work : sms;
  const int pages_avail = (pos0 + T + BI_PAGE_TOKENS - 1) / BI_PAGE_TOKENS;
  const int32_t* prow = page_table + (int64_t)seq * max_pages_per_seq;
  const float c = (float)((double)scale * 1.4426950408889634);
  cudaStream_t st = as_stream(stream);
  static std::once_flag once[2][64];
  static cudaError_t attr[2][64];
  if (D == 128) {
    if (bi::gemm::set_smem_once(bi::attn_tc::prefill_tc_kernel<128>, bi::attn_tc::Cfg<128>::SMEM, once[0], attr[0],
                                dev) != cudaSuccess)
      return BI_ERR_CUDA;
    bi::attn_tc::prefill_tc_kernel<128><<<grid, bi::attn_tc::kThreads, bi::attn_tc::Cfg<128>::SMEM, st>>>(
        tq, tk, tv, prow, num_pages, Hq, Hkv, pos0, T, pages_avail, out, c);
  } else {
    if (bi::gemm::set_smem_once(bi::attn_tc::prefill_tc_kernel<64>, bi::attn_tc::Cfg<64>::SMEM, once[1], attr[1],
                                dev) != cudaSuccess)
      return BI_ERR_CUDA;
    bi::attn_tc::prefill_tc_kernel<64><<<grid, bi::attn_tc::kThreads, bi::attn_tc::Cfg<64>::SMEM, st>>>(
        tq, tk, tv, prow, num_pages, Hq, Hkv, pos0, T, pages_avail, out, c);
  }
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status bi_kv_append(const bi_bf16* k_new, const bi_bf16* v_new, int64_t ld_new, const int32_t* q_seq, const int32_t* q_pos,
                       bi_bf16* k_cache, bi_bf16* v_cache, int64_t num_pages, const int32_t* page_table,
                       int num_seqs, int max_pages_per_seq, int T, int Hkv, int D, void* stream) {
  if (!k_new || !v_new || !q_seq || !q_pos || !k_cache || !v_cache || !page_table) return BI_ERR_NULL;
  if (T < 0 || num_seqs <= 0 || max_pages_per_seq <= 0 || num_pages <= 0 || Hkv <= 0 || D <= 0)
    return BI_ERR_SHAPE;
  if (D % 8 != 0) return BI_ERR_UNSUPPORTED;
  if (ld_new < (int64_t)Hkv * D) return BI_ERR_SHAPE;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) || ld_new % 8)
    return BI_ERR_ALIGN;
  if (T == 0) return BI_OK;
  const int64_t warps = (int64_t)T * Hkv;
  if ((warps + 7) / 8 > INT_MAX) return BI_ERR_SHAPE;
  return bi::launch_pdl(bi::attn::kv_append_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, as_stream(stream),
                        k_new, v_new, ld_new, q_seq, q_pos, k_cache, v_cache, num_pages, page_table, num_seqs,
                        max_pages_per_seq, T, Hkv, D) == cudaSuccess
             ? BI_OK
             : BI_ERR_CUDA;
}

size_t bi_lmhead_workspace_size(int64_t M, int64_t V) { return lm_ws_size(M, V, nullptr, nullptr); }

bi_status bi_lmhead_argmax(const bi_bf16* h, int64_t ldh, const bi_bf16* W, int64_t M, int64_t V, int64_t K,
                           float margin_threshold, int32_t* tokens, int32_t* recomputed, float* logits_fp32,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!h || !W || !tokens || !recomputed) return BI_ERR_NULL;
  if (M < 0 || V < 8 || V % 8 != 0 || K < 64 || K % 64 != 0 || ldh < K || M > INT_MAX || V > INT_MAX ||
      std::isnan(margin_threshold))
    return BI_ERR_SHAPE;
  if (!aligned16(h) || !aligned16(W) || ldh % 8 || (logits_fp32 && !aligned16(logits_fp32))) return BI_ERR_ALIGN;
  if (M == 0) return BI_OK;
  if (!workspace) return BI_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BI_ERR_ALIGN;
  if ((M + 31) / 32 > 65535) return BI_ERR_UNSUPPORTED;
  LmWs lay{};
  if (workspace_bytes < lm_ws_size(M, V, &lay, workspace)) return BI_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BI_ERR_CUDA;
  bi_status s = bi::gemm::launch(h, ldh, W, K, lay.logits16, V, M, V, K, st);
  if (s != BI_OK) return s;
  // small batches (M <= 24, hidden size <= 4096): the streaming recompute lists the
  // flagged rows and takes their tokens itself; W is streamed once for a single flagged
  // row, once per group of 8 otherwise. Larger batches: the flagged list, then 64-row
  // tiles and a separate argmax. Every fp32 logit is the same FMA chain on each path;
  // each kernel returns at once when the flagged count (known on the device) is not
  // its case.
  const bool small = M <= bi::lmhead::kStrMaxCount && K <= bi::lmhead::kStrMaxK;
  if (bi::launch_pdl(bi::lmhead::top2_kernel, dim3((unsigned)(M * bi::lmhead::kParts)), dim3(bi::lmhead::kThreads), 0,
                     st, (const uint16_t*)lay.logits16, V, margin_threshold, tokens, recomputed,
                     small ? lay.ticket : (unsigned int*)nullptr) != cudaSuccess)
    return BI_ERR_CUDA;
  float* out32 = logits_fp32 ? logits_fp32 : lay.logits32;
  if (small) {
    static std::once_flag once_str[64];
    static cudaError_t attr_str[64];
    if (bi::gemm::set_smem_once(bi::lmhead::recompute_stream_kernel, bi::lmhead::stream_smem_bytes(bi::lmhead::kStrMaxK),
                                once_str, attr_str, dev) != cudaSuccess)
      return BI_ERR_CUDA;
    const unsigned sgrid = (unsigned)((V + bi::lmhead::kStrWarps * 32 - 1) / (bi::lmhead::kStrWarps * 32));
    const cudaError_t e = bi::launch_pdl(bi::lmhead::recompute_stream_kernel, dim3(sgrid), dim3(bi::lmhead::kStrThreads),
                                         (size_t)bi::lmhead::stream_smem_bytes((int)K), st, h, ldh, W, V, (int)K,
                                         (int)M, (const int32_t*)recomputed, out32, lay.arg_part, tokens, lay.ticket);
    return e == cudaSuccess ? BI_OK : BI_ERR_CUDA;
  }
  cudaError_t e = bi::launch_pdl(bi::lmhead::compact_kernel, dim3(1), dim3(1024), 0, st, (const int32_t*)recomputed,
                                 (int)M, lay.list);
  const dim3 rgrid((unsigned)((V + bi::lmhead::VB - 1) / bi::lmhead::VB),
                   (unsigned)((M + bi::lmhead::RB - 1) / bi::lmhead::RB));
  if (e == cudaSuccess)
    e = bi::launch_pdl(bi::lmhead::recompute_kernel, rgrid, dim3(bi::lmhead::kRecThreads), 0, st, h, ldh, W, V, (int)K,
                       (int)M, (const int32_t*)lay.list, out32, 0);
  if (e == cudaSuccess)
    e = bi::launch_pdl(bi::lmhead::argmax_kernel, dim3((unsigned)(M * bi::lmhead::kParts)), dim3(bi::lmhead::kThreads),
                       0, st, (const float*)out32, V, (const int32_t*)recomputed, tokens);
  return e == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status bi_gather_rows(const bi_bf16* src, int64_t ld_src, int64_t nrows_src, const int32_t* idx, int64_t M,
                         int64_t width, bi_bf16* dst, int64_t ld_dst, void* stream) {
  if (!src || !idx || !dst) return BI_ERR_NULL;
  if (M < 0 || nrows_src <= 0 || width <= 0 || width % 8 || ld_src < width || ld_dst < width || M > INT_MAX)
    return BI_ERR_SHAPE;
  if (!aligned16(src) || !aligned16(dst) || ld_src % 8 || ld_dst % 8) return BI_ERR_ALIGN;
  if (M == 0) return BI_OK;
  return bi::launch_pdl(bi::glue::gather_rows_kernel, dim3((unsigned)((M + 7) / 8)), dim3(256), 0, as_stream(stream),
                        src, ld_src, nrows_src, idx, (int)M, width, dst, ld_dst) == cudaSuccess
             ? BI_OK
             : BI_ERR_CUDA;
}

bi_status bi_rope(bi_bf16* x, int64_t ldx, int64_t T, int H, int D, const int32_t* pos, const float* cos_sin,
                  int max_pos, void* stream) {
  if (!x || !pos || !cos_sin) return BI_ERR_NULL;
  if (T < 0 || T > INT_MAX || H <= 0 || D <= 0 || D % 2 || max_pos <= 0 || ldx < (int64_t)H * D)
    return BI_ERR_SHAPE;
  if (T == 0) return BI_OK;
  const int64_t n = T * H * (D / 2);
  if ((n + 255) / 256 > INT_MAX) return BI_ERR_SHAPE;
  return bi::launch_pdl(bi::glue::rope_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, as_stream(stream), x,
                        ldx, (int)T, H, D, pos, reinterpret_cast<const float2*>(cos_sin), max_pos) == cudaSuccess
             ? BI_OK
             : BI_ERR_CUDA;
}

bi_status bi_swiglu(const bi_bf16* gate_up, int64_t ld_gu, bi_bf16* out, int64_t ld_out, int64_t M, int64_t F,
                    void* stream) {
  if (!gate_up || !out) return BI_ERR_NULL;
  if (M < 0 || F <= 0 || F % 8 || ld_gu < 2 * F || ld_out < F) return BI_ERR_SHAPE;
  if (!aligned16(gate_up) || !aligned16(out) || ld_gu % 8 || ld_out % 8) return BI_ERR_ALIGN;
  if (M == 0) return BI_OK;
  const int64_t n = M * (F / 8);
  if ((n + 255) / 256 > INT_MAX || M > INT_MAX) return BI_ERR_SHAPE;
  return bi::launch_pdl(bi::glue::swiglu_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, as_stream(stream),
                        gate_up, ld_gu, out, ld_out, (int)M, (int)F) == cudaSuccess
             ? BI_OK
             : BI_ERR_CUDA;
}

bi_status bi_add(const bi_bf16* a, const bi_bf16* b, bi_bf16* out, int64_t n, void* stream) {
  if (!a || !b || !out) return BI_ERR_NULL;
  if (n < 0 || n % 8) return BI_ERR_SHAPE;
  if (!aligned16(a) || !aligned16(b) || !aligned16(out)) return BI_ERR_ALIGN;
  if (n == 0) return BI_OK;
  const int64_t v = n / 8;
  if ((v + 255) / 256 > INT_MAX) return BI_ERR_SHAPE;
  return bi::launch_pdl(bi::glue::add_kernel, dim3((unsigned)((v + 255) / 256)), dim3(256), 0, as_stream(stream), a, b,
                        out, n) == cudaSuccess
             ? BI_OK
             : BI_ERR_CUDA;
}

bi_status bi_selftest_wait_timeout(int limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 2000) return BI_ERR_SHAPE;
  bi::selftest_wait_kernel<<<1, 1, 0, as_stream(stream)>>>((uint64_t)limit_ms * 1000000ull);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status bi_get_device_error(int32_t* code) {
  if (!code) return BI_ERR_NULL;
  if (cudaDeviceSynchronize() != cudaSuccess) return BI_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, bi::g_error_word, sizeof(int)) != cudaSuccess) return BI_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(bi::g_error_word, &zero, sizeof(int)) != cudaSuccess) return BI_ERR_CUDA;
  *code = v;
  return BI_OK;
}

// ---- row reductions and sampling

namespace {

bi_status rows_check(const void* x, int64_t ldx, int64_t M, int64_t N) {
  if (M < 0 || M > INT_MAX || N < 8 || N % 8 != 0 || N > (int64_t(1) << 24) || ldx < N) return BI_ERR_SHAPE;
  if (!aligned16(x) || ldx % 8) return BI_ERR_ALIGN;
  return BI_OK;
}

}  // namespace

bi_status bi_log_softmax(const bi_bf16* x, int64_t ldx, float* y, int64_t ldy, int64_t M, int64_t N,
                         void* stream) {
  if (!x || !y) return BI_ERR_NULL;
  if (bi_status e = rows_check(x, ldx, M, N)) return e;
  if (ldy < N) return BI_ERR_SHAPE;
  if (!aligned16(y) || ldy % 4) return BI_ERR_ALIGN;
  if (M == 0) return BI_OK;
  if (ranges_overlap(x, span_bytes(M, N, ldx, 2), y, span_bytes(M, N, ldy, 4))) return BI_ERR_SHAPE;
  BI_RED_DISPATCH(bi::red::log_softmax_kernel, N, (unsigned)M, as_stream(stream), x, ldx, y, ldy, (int)N);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status bi_token_logprob(const bi_bf16* x, int64_t ldx, const int32_t* tokens, float* out, int64_t M,
                           int64_t N, void* stream) {
  if (!x || !tokens || !out) return BI_ERR_NULL;
  if (bi_status e = rows_check(x, ldx, M, N)) return e;
  if (M == 0) return BI_OK;
  BI_RED_DISPATCH(bi::red::token_logprob_kernel, N, (unsigned)M, as_stream(stream), x, ldx, tokens, out, (int)N);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status bi_row_mean(const bi_bf16* x, int64_t ldx, float* y, int64_t M, int64_t K, void* stream) {
  if (!x || !y) return BI_ERR_NULL;
  if (bi_status e = rows_check(x, ldx, M, K)) return e;
  if (M == 0) return BI_OK;
  BI_RED_DISPATCH(bi::red::row_mean_kernel, K, (unsigned)M, as_stream(stream), x, ldx, y, (int)K);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status bi_sampling_uniforms(const uint64_t* seeds, const uint64_t* steps, float* u, int64_t ldu, int64_t M,
                               int64_t V, void* stream) {
  if (!seeds || !steps || !u) return BI_ERR_NULL;
  if (M < 0 || M > INT_MAX || V < 8 || V % 8 != 0 || V > (int64_t(1) << 24) || ldu < V) return BI_ERR_SHAPE;
  if (!aligned16(u) || ldu % 4) return BI_ERR_ALIGN;
  if (M == 0) return BI_OK;
  bi::red::uniforms_kernel<<<(unsigned)M, bi::red::kThreads, 0, as_stream(stream)>>>(seeds, steps, u, ldu, (int)V);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status bi_sample(const bi_bf16* logits, int64_t ld, const uint64_t* seeds, const uint64_t* steps,
                    float temperature, int32_t* tokens, int64_t M, int64_t V, void* stream) {
  if (!logits || !seeds || !steps || !tokens) return BI_ERR_NULL;
  if (bi_status e = rows_check(logits, ld, M, V)) return e;
  if (M > INT_MAX / bi::red::kSampleParts) return BI_ERR_SHAPE;
  if (!std::isfinite(temperature) || !(temperature > 0.f)) return BI_ERR_SHAPE;
  const float inv_t = 1.0f / temperature;  // IEEE division: 1/T rounded once
  if (!std::isfinite(inv_t)) return BI_ERR_SHAPE;
  if (M == 0) return BI_OK;
  bi::red::sample_kernel<<<(unsigned)(M * bi::red::kSampleParts), bi::red::kThreads, 0, as_stream(stream)>>>(
      logits, ld, seeds, steps, inv_t, tokens, (int)V);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

}  // extern "C"
