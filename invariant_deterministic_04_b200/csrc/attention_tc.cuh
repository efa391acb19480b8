// Causal prefill attention on 5th-generation tensor cores, batch- and chunk-invariant.
//
// Source: "Defeating Nondeterminism in LLM Inference" technical summary
// (mobiles-han blog), section 対応策：バッチ不変なカーネル設計, kernel table, row
// Attention (one layout for cache and chunk; a schedule that does not depend on the
// chunking), and the French article's "Le prix d'une sortie bit à bit identique"
// section (a faster attention kernel recovers most of the cost: 55 s -> 42 s).
//
// One chunk of one sequence: query rows at positions pos0 .. pos0 + T - 1, keys
// 0 .. pos from the paged store (the chunk's own K/V already appended).
// Per-row schedule, a function of the row's position only:
//   * keys are processed in blocks of 64 at absolute positions 0, 64, 128, ..., in
//     ascending order, up to the block holding the row's position;
//   * S = q . k for a block by tcgen05.mma (bf16 x bf16, fp32 accumulation over D in
//     ascending 16-wide steps), masked to keys <= pos;
//   * online softmax in fp32 by the thread that owns the row: b = block max of the
//     masked q.k times c (c = scale * log2 e); the reference point m becomes b only
//     when b > m + 8 (lazy rescaling: p stays <= 2^8, exact in fp32, and the final
//     division by l cancels the choice of m); p_j = 2^(q.k_j * c - m) (one FMA, one
//     SFU exp2); l = l * 2^(m_old - m) + the block's p summed as eight partial sums
//     (key index mod 8, keys in order) joined by a fixed tree; O rescaled by
//     2^(m_old - m) only when m moved (x * 1 == x);
//   * p rounded to bf16, O += P V by tcgen05.mma (fp32, ascending 16-key steps);
//   * out = O * (1 / l) rounded to bf16.
// The tensor core's result for an output element depends on that element's row and
// column operands and the fixed K order only, not on the other rows of the tile or
// the tile shape (checked on this hardware by the matmul tests), and a block with
// no visible key leaves a row's state unchanged; so a row's bits do not depend on
// how the sequence was chunked or which other rows shared its tile.
//
// Work: a CTA takes two 128-row Q tiles at once, query heads h and h+1 of one kv-head
// over the same row block, so every K/V block is fetched once for both. Warp 0 loads
// (TMA), warp 1 issues the MMAs in a software pipeline (S of one tile while the
// other tile's softmax runs), warps 2-5 and 6-9 run the two softmaxes.
#pragma once

#include "device.cuh"

namespace bi {
namespace attn_tc {

constexpr int PAGE = BI_PAGE_TOKENS;
constexpr int KB = 64;                  // keys per block
constexpr int PAGES_PER_BLOCK = KB / PAGE;
constexpr int ROWS = 128;               // query rows per tile
constexpr int kThreads = 320;           // warp 0 TMA, warp 1 MMA, warps 2-5 / 6-9 softmax of tiles A / B
constexpr float kLazy = 8.f;            // the softmax reference point moves by more than 2^8 or not at all

template <int D>
struct Cfg {
  static constexpr int HALVES = D / 64;                 // 64-dim (128-byte) halves
  static constexpr int Q_BYTES = ROWS * D * 2;          // one Q tile
  static constexpr int KV_HALF = KB * 128;              // one 64-dim half of a 64-key block
  static constexpr int K_BYTES = HALVES * KV_HALF;
  static constexpr int STAGE = 2 * K_BYTES;             // K and V of one block
  static constexpr int P_BYTES = ROWS * KB * 2;         // one P tile (bf16, 128-byte rows)
  static constexpr int STAGES = 3;
  static constexpr int SMEM = 1024 + 2 * Q_BYTES + STAGES * STAGE + 2 * P_BYTES + 256;
  static constexpr int TMEM_COLS = (2 * KB + 2 * D) <= 256 ? 256 : 512;  // S_A, S_B, O_A, O_B
};

// Instruction descriptors (kind::f16, bf16 inputs, fp32 accumulate, M = 128).
// S = Q K^T: A = Q K-major, B = K K-major, N = 64 keys.
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(KB >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
// O += P V: A = P K-major (keys contiguous), B = V MN-major (dims contiguous), N = D.
template <int D>
__host__ __device__ constexpr uint32_t idesc_pv() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(D >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// K-major, 128-byte swizzle: 128-byte rows, 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// MN-major, 128-byte swizzle: 64 MN elements per 128-byte row, K rows 128 bytes
// apart, 8-K-row groups 1024 bytes apart (SBO), 64-element MN chunks lbo bytes apart.
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// 2^x by the SFU (one instruction; 2^-inf = +0, subnormal results flushed to zero).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ page_row,
                      int64_t num_pages, int Hq, int Hkv, int pos0, int T, int pages_avail,
                      uint16_t* __restrict__ out, float c) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t q_s = base;                            // tile X at q_s + X * Q_BYTES
  const uint32_t kv_s = base + 2 * C::Q_BYTES;          // stage s: K at kv_s + s*STAGE, V at + K_BYTES
  const uint32_t p_s = kv_s + C::STAGES * C::STAGE;     // tile X at p_s + X * P_BYTES
  const uint32_t bar0 = p_s + 2 * C::P_BYTES;
  // barriers: Q_FULL, Q_EMPTY, KV_FULL[s], KV_EMPTY[s], then per tile X: S_FULL, P_FULL, O_DONE, O_FREE
  const uint32_t Q_FULL = bar0, Q_EMPTY = bar0 + 8;
  auto KV_FULL = [&](int s) { return bar0 + 16 + 16 * s; };
  auto KV_EMPTY = [&](int s) { return bar0 + 24 + 16 * s; };
  const uint32_t XB = bar0 + 16 + 16 * C::STAGES;
  auto S_FULL = [&](int x) { return XB + 32 * x; };
  auto P_FULL = [&](int x) { return XB + 32 * x + 8; };
  auto O_DONE = [&](int x) { return XB + 32 * x + 16; };
  auto O_FREE = [&](int x) { return XB + 32 * x + 24; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + (XB - base) + 64);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = Hq / Hkv;
  const int pairs = Hkv * (G / 2);                      // tile pairs per row block
  const int rblocks = (T + ROWS - 1) / ROWS;
  const int work = rblocks * pairs;

  if (threadIdx.x == 0) {
    mbar_init(Q_FULL, 1);
    mbar_init(Q_EMPTY, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(KV_FULL(s), 1);
      mbar_init(KV_EMPTY(s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(S_FULL(x), 1);
      mbar_init(P_FULL(x), 128);
      mbar_init(O_DONE(x), 1);
      mbar_init(O_FREE(x), 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the producer's filled stages and their phase parities (Q, and the K/V ring)
  uint32_t q_issued = 0, q_ph_bits = 0, kv_issued = 0, kv_ph_bits = 0;
  auto tS = [&](int x) { return tmem + (uint32_t)(x * KB); };
  auto tO = [&](int x) { return tmem + (uint32_t)(2 * KB + x * D); };

  // work item w -> (kv-head g, first query head hA = g*G + 2*hp, row block rb);
  // heavier row blocks (more key blocks) first
  auto item_of = [&](int w, int& g, int& hA, int& rb) {
    rb = rblocks - 1 - w / pairs;
    const int pr = w % pairs;
    g = pr / (G / 2);
    hA = g * G + 2 * (pr % (G / 2));
  };
  // the CTA's k-th item: rounds of gridDim.x items in snake order (items are sorted
  // heaviest first, so alternate rounds hand the lightest to the CTAs that got the heaviest)
  auto item_at = [&](int k) {
    return k * (int)gridDim.x + ((k & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
  };
  auto nblocks_of = [&](int rb) {
    const int last_row = min(T, (rb + 1) * ROWS) - 1;
    return (pos0 + last_row) / KB + 1;
  };

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer
      int s = 0;
      uint32_t ph = 0, qph = 0;
      for (int k = 0, w = item_at(0); w < work && !*abort_flag; w = item_at(++k)) {
        int g, hA, rb;
        item_of(w, g, hA, rb);
        if (!mbar_wait(Q_EMPTY, qph ^ 1u)) { *abort_flag = 1; break; }
        qph ^= 1u;
        mbar_arrive_expect_tx(Q_FULL, 2 * C::Q_BYTES);
        for (int x = 0; x < 2; ++x)
          for (int hh = 0; hh < C::HALVES; ++hh)
            tma_load_2d(q_s + x * C::Q_BYTES + hh * (ROWS * 128), &tmQ, (hA + x) * D + hh * 64, rb * ROWS, Q_FULL);
        note_fill(q_issued, q_ph_bits, 0, qph ^ 1u);
        const int nb = nblocks_of(rb);
        bool ok = true;
        for (int j = 0; j < nb; ++j) {
          if (!mbar_wait(KV_EMPTY(s), ph ^ 1u)) { ok = false; break; }
          int np = pages_avail - j * PAGES_PER_BLOCK;
          np = np < 0 ? 0 : (np > PAGES_PER_BLOCK ? PAGES_PER_BLOCK : np);
          int valid_pages = 0;
          for (int p = 0; p < np; ++p) {
            const int pg = page_row[j * PAGES_PER_BLOCK + p];
            if (pg >= 0 && pg < num_pages) ++valid_pages;
            else record_error(BI_ERR_DEVICE_INDEX);
          }
          mbar_arrive_expect_tx(KV_FULL(s), (uint32_t)(valid_pages * PAGE * D * 2 * 2));
          const uint32_t ks = kv_s + s * C::STAGE, vs = ks + C::K_BYTES;
          for (int p = 0; p < np; ++p) {
            const int pg = page_row[j * PAGES_PER_BLOCK + p];
            if (pg < 0 || pg >= num_pages) continue;
            const int row = (pg * Hkv + g) * PAGE;  // first row of this page in the [pages*Hkv*16, D] view
            for (int hh = 0; hh < C::HALVES; ++hh) {
              tma_load_2d(ks + hh * C::KV_HALF + p * (PAGE * 128), &tmK, hh * 64, row, KV_FULL(s));
              tma_load_2d(vs + hh * C::KV_HALF + p * (PAGE * 128), &tmV, hh * 64, row, KV_FULL(s));
            }
          }
          note_fill(kv_issued, kv_ph_bits, s, ph);
          if (++s == C::STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) { *abort_flag = 1; break; }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer (software-pipelined over the two tiles)
      int s = 0;
      uint32_t ph = 0, qph = 0;
      uint32_t pph[2] = {0, 0}, oph[2] = {0, 0};
      bool ok = true;
      auto issue_s = [&](int x, int st) {
        const uint32_t ks = kv_s + st * C::STAGE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = x * C::Q_BYTES + (kk / 4) * (ROWS * 128) + (kk % 4) * 32;
          const uint32_t koff = (kk / 4) * C::KV_HALF + (kk % 4) * 32;
          tc_mma_f16(tS(x), desc_k(q_s + qoff), desc_k(ks + koff), kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit(S_FULL(x));
      };
      auto issue_pv = [&](int x, int st, int j) {
        const uint32_t vs = kv_s + st * C::STAGE + C::K_BYTES;
#pragma unroll
        for (int kk = 0; kk < KB / 16; ++kk)
          tc_mma_f16(tO(x), desc_k(p_s + x * C::P_BYTES + kk * 32), desc_mn(vs + kk * (16 * 128), C::KV_HALF),
                     idesc_pv<D>(), (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(O_DONE(x));
      };
      for (int k = 0, w = item_at(0); w < work && ok && !*abort_flag; w = item_at(++k)) {
        int g, hA, rb;
        item_of(w, g, hA, rb);
        const int nb = nblocks_of(rb);
        if (!mbar_wait(Q_FULL, qph)) { ok = false; break; }
        qph ^= 1u;
        // prologue: S of block 0 for both tiles
        if (!mbar_wait(KV_FULL(s), ph)) { ok = false; break; }
        tc_fence_after();
        issue_s(0, s);
        issue_s(1, s);
        for (int j = 0; j < nb && ok; ++j) {
          const int sj = s;
          const int sn = (s + 1 == C::STAGES) ? 0 : s + 1;
          const uint32_t phn = (s + 1 == C::STAGES) ? (ph ^ 1u) : ph;
          for (int x = 0; x < 2 && ok; ++x) {
            if (j == 0) {  // the previous tile's O of this group has been read out
              if (!mbar_wait(O_FREE(x), oph[x] ^ 1u)) { ok = false; break; }
              oph[x] ^= 1u;
            }
            if (!mbar_wait(P_FULL(x), pph[x])) { ok = false; break; }
            pph[x] ^= 1u;
            tc_fence_after();
            issue_pv(x, sj, j);
            if (x == 1) tc_commit(KV_EMPTY(sj));  // both tiles are done with block j
            if (j + 1 < nb) {
              if (x == 0 && !mbar_wait(KV_FULL(sn), phn)) { ok = false; break; }
              tc_fence_after();
              issue_s(x, sn);
            }
          }
          s = sn;
          ph = phn;
        }
        if (!ok) break;
        tc_commit(Q_EMPTY);  // all S of this tile pair were issued before this point
      }
      if (!ok) *abort_flag = 1;
    }
  } else {  // ---- softmax: warps 2..5 (tile A) and 6..9 (tile B); thread = query row (TMEM lane)
    const int x = (warp - 2) / 4;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row within the tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    uint32_t sph = 0, oph = 0, kvph = 0;
    int s = 0;
    bool ok = true;
    for (int k = 0, w = item_at(0); w < work; w = item_at(++k)) {
      int g, hA, rb;
      item_of(w, g, hA, rb);
      const int h = hA + x;
      const int nb = nblocks_of(rb);
      const int row = rb * ROWS + r;               // row within the chunk
      const int pos = pos0 + (row < T ? row : T - 1);
      const int max_pos = pos0 + min(T, (rb + 1) * ROWS) - 1;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nb; ++j) {
        ok = __all_sync(kFullMask, mbar_wait(S_FULL(x), sph));
        if (!ok) break;
        sph ^= 1u;
        tc_fence_after();
        const int key0 = j * KB;
        // every key of the block visible to every row of this warp: no masking needed
        const bool full = __all_sync(kFullMask, key0 + KB - 1 <= pos);
        // the block's 64 scores of this row, read from tensor memory once; masked keys
        // become -inf (NaN of stale slots never survives the select)
        uint32_t sv[KB];
        __syncwarp();
        tmem_ld_32x32b_x32(tS(x) + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld_32x32b_x32(tS(x) + lane_base + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
        if (!full) {
#pragma unroll
          for (int e = 0; e < KB; ++e)
            if (key0 + e > pos) sv[e] = __float_as_uint(-INFINITY);
        }
        float bm[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) bm[e] = -INFINITY;
#pragma unroll
        for (int e = 0; e < KB; ++e) bm[e & 7] = fmaxf(bm[e & 7], __uint_as_float(sv[e]));
        const float bmax =
            fmaxf(fmaxf(fmaxf(bm[0], bm[1]), fmaxf(bm[2], bm[3])), fmaxf(fmaxf(bm[4], bm[5]), fmaxf(bm[6], bm[7])));
        // the reference point m moves only when the block max exceeds it by more than 2^8;
        // scores up to 256 * 2^m stay exact in fp32 and the final 1/l cancels the choice
        const float sb = __fmul_rn(bmax, c);  // scores are q.k * c with c > 0
        const bool move = sb > __fadd_rn(m, kLazy);
        const float m_new = move ? sb : m;
        const float alpha = (move && m != -INFINITY) ? ex2_approx(__fsub_rn(m, m_new)) : 1.f;
        const float2 neg_m2 = make_float2(-m_new, -m_new);
        const float2 c2 = make_float2(c, c);
        // the previous P . V of this tile must be done before P is overwritten and O rescaled
        if (j > 0) {
          ok = __all_sync(kFullMask, mbar_wait(O_DONE(x), oph));
          if (!ok) break;
          oph ^= 1u;
          tc_fence_after();
        }
        // p = 2^(q.k * c - m) (masked keys give 2^-inf = 0), partial sums by key
        // index mod 8, P row as bf16 into the swizzled 128-byte row
        float2 ps[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) ps[e] = make_float2(0.f, 0.f);
#pragma unroll
        for (int cc = 0; cc < KB / 32; ++cc) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 t = __ffma2_rn(make_float2(__uint_as_float(sv[cc * 32 + q8 * 8 + 2 * e]),
                                                      __uint_as_float(sv[cc * 32 + q8 * 8 + 2 * e + 1])),
                                          c2, neg_m2);
              const float2 pv = make_float2(ex2_approx(t.x), ex2_approx(t.y));
              ps[e] = __fadd2_rn(ps[e], pv);
              pk[e] = pack_bf16x2(pv.x, pv.y);
            }
            const int chunk = cc * 4 + q8;
            st_shared_v4(p_s + x * C::P_BYTES + r * 128 + ((chunk ^ (r & 7)) << 4),
                         make_uint4(pk[0], pk[1], pk[2], pk[3]));
          }
        }
        const float psum = __fadd_rn(__fadd_rn(__fadd_rn(ps[0].x, ps[0].y), __fadd_rn(ps[1].x, ps[1].y)),
                                     __fadd_rn(__fadd_rn(ps[2].x, ps[2].y), __fadd_rn(ps[3].x, ps[3].y)));
        l = __fadd_rn(__fmul_rn(l, alpha), psum);
        if (j > 0 && __any_sync(kFullMask, alpha != 1.f)) {
          // rescale this warp's rows of O in tensor memory (rows with alpha == 1 are unchanged)
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t ov[32];
            __syncwarp();
            tmem_ld_32x32b_x32(tO(x) + lane_base + cc * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__fmul_rn(__uint_as_float(ov[e]), alpha));
            tmem_st_32x32b_x32(tO(x) + lane_base + cc * 32, ov);
          }
          tmem_wait_st();
        }
        m = m_new;
        // V rows of keys past the chunk may be stale (even NaN): tile A's group zeroes them
        // before P . V (tile B's P . V is issued after tile A's)
        if (x == 0) {
          const int stage = s;
          (void)mbar_wait(KV_FULL(stage), kvph);  // already complete: acquires the TMA writes
          const int valid = max_pos + 1 - key0;
          if (valid < KB && r < KB && r >= valid) {
            const uint32_t vs = kv_s + stage * C::STAGE + C::K_BYTES;
            for (int hh = 0; hh < C::HALVES; ++hh)
              for (int ch = 0; ch < 8; ++ch) st_shared_v4(vs + hh * C::KV_HALF + r * 128 + ch * 16, make_uint4(0, 0, 0, 0));
          }
        }
        if (++s == C::STAGES) { s = 0; kvph ^= 1u; }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(P_FULL(x));
      }
      if (!ok) break;
      // final O / l for this tile
      ok = __all_sync(kFullMask, mbar_wait(O_DONE(x), oph));
      if (!ok) break;
      oph ^= 1u;
      tc_fence_after();
      uint16_t* dst = out + ((int64_t)row * Hq + h) * D;
      const float inv_l = __frcp_rn(l);
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ov[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tO(x) + lane_base + cc * 32, ov);
        tmem_wait_ld();
        if (row < T) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 o;
            o.x = pack_bf16x2(__fmul_rn(__uint_as_float(ov[8 * v + 0]), inv_l), __fmul_rn(__uint_as_float(ov[8 * v + 1]), inv_l));
            o.y = pack_bf16x2(__fmul_rn(__uint_as_float(ov[8 * v + 2]), inv_l), __fmul_rn(__uint_as_float(ov[8 * v + 3]), inv_l));
            o.z = pack_bf16x2(__fmul_rn(__uint_as_float(ov[8 * v + 4]), inv_l), __fmul_rn(__uint_as_float(ov[8 * v + 5]), inv_l));
            o.w = pack_bf16x2(__fmul_rn(__uint_as_float(ov[8 * v + 6]), inv_l), __fmul_rn(__uint_as_float(ov[8 * v + 7]), inv_l));
            reinterpret_cast<uint4*>(dst + cc * 32)[v] = o;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(O_FREE(x));
    }
    if (!ok) *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  // after an abort, loads may still be landing in stages nobody waited for
  if (warp == 0 && lane == 0 && *abort_flag) {
    drain_copies(Q_FULL, 8, q_issued, q_ph_bits);
    drain_copies(KV_FULL(0), 16, kv_issued, kv_ph_bits);
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn_tc
}  // namespace bi
